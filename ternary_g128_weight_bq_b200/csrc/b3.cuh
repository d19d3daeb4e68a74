// b3.cuh -- the base-3 ternary storage (BQ_TERNARY_B3_G128): where each code of a group sits and
// how a byte turns back into codes.
//
// Ternary Bonsai 27B article (wmrh.cn), section "局限性与未来发展": the deployed ternary weights
// use 2-bit storage although their information is 1.71 bits per weight, and native ternary
// kernels are still to come. This library's base-3 layout (the pages fix none):
//   * codes c = value + 1 in {0, 1, 2}; a group of 128 takes 26 bytes: bytes 0..23 hold five
//     codes (group positions 5j .. 5j+4), bytes 24 and 25 four codes (120..123, 124..127);
//   * a byte holding n codes stores ceil(256 v / 3^n), v = the codes as a base-3 number with the
//     first code most significant: an 8-bit fixed-point fraction, rounded up, of v / 3^n;
//   * a row is a run of blocks of 8 groups (the last may hold fewer, nb): first the 24 five-code
//     bytes of each group (group i at 24 i), then the two four-code bytes of each (at 24 nb + 2 i).
//     A full block is 208 bytes, a row 26 K / 128: 1.75 bits per weight with the fp16 scale.
//
// Decoding. With q the stored byte, F_i = floor(q 3^i / 256) (i = 1 .. n) is the number formed
// by the first i codes, so code p is F_{p+1} - 3 F_p (F_0 = 0): each level costs one multiply by
// a constant and a byte extraction, and q 3^5 < 2^16 lets two bytes share one 32-bit multiply in
// 16-bit lanes. (q = ceil(256 v / 3^n) = 256 v / 3^n + d with 0 <= d < 1, so q 3^i / 256 exceeds
// v / 3^(n-i) by less than 3^(i-n), which never reaches the next integer.)
#pragma once

#include <stdint.h>

namespace bq {
namespace b3 {

constexpr int kGroupBytes = 26;
constexpr int kBlockBytes = 8 * kGroupBytes;     // 208

__host__ __device__ constexpr int count(int j) { return j < 24 ? 5 : 4; }
__host__ __device__ constexpr int first(int j) { return j < 24 ? 5 * j : 120 + 4 * (j - 24); }
__host__ __device__ constexpr int byte_of(int kk) { return kk < 120 ? kk / 5 : 24 + (kk - 120) / 4; }
__host__ __device__ constexpr uint32_t pow3(int i)
{
    return i <= 0 ? 1u : i == 1 ? 3u : i == 2 ? 9u : i == 3 ? 27u : i == 4 ? 81u : 243u;
}

// Offset within a row of G groups of byte j of group g.
__host__ __device__ inline int64_t byte_offset(int64_t G, int64_t g, int j)
{
    const int64_t f = g & ~int64_t(7);                 // first group of g's block
    const int64_t nb = G - f < 8 ? G - f : 8;
    return j < 24 ? kGroupBytes * f + 24 * (g - f) + j : kGroupBytes * f + 24 * nb + 2 * (g - f) + (j - 24);
}

// The byte written for n codes of base-3 value v (0 <= v < 3^n).
__host__ __device__ inline uint32_t encode(uint32_t v, int n) { return (256u * v + pow3(n) - 1u) / pow3(n); }

// Code p of a byte q holding n codes; -1 if q is not a byte the encoding writes.
__device__ __forceinline__ int code(uint32_t q, int n, int p)
{
    const uint32_t v = (q * pow3(n)) >> 8;
    if (encode(v, n) != q)
        return -1;
    return (int)(((q * pow3(p + 1)) >> 8) - 3u * ((q * pow3(p)) >> 8));
}

}  // namespace b3
}  // namespace bq
