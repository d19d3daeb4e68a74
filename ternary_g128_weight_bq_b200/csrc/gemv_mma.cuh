// gemv_mma.cuh -- the integer tensor-core arithmetic shared by the decode GEMV kernels
// (mma.sync m16n8k32 s8): how sign bits / ternary codes become s8 A operands, how x becomes
// balanced integer digits in the B operand, and the fragment layout both sides agree on.
//
// Model card "prism-ml/Bonsai-27B-mlx-1bit", sections "Weight representation: Binary g128" and
// "CUDA (NVIDIA GPUs)": y[m][n] = sum_g s[n][g] * sum_{k in g} v[n][k] x[m][k], v = +-1 (binary)
// or {-1, 0, +1} (ternary: "Ternary Bonsai 27B vs ..." article, wmrh.cn).
//
// x as integers. Per (token, group of 128), x is written as X = round(x * 2^(21-e)) with
// e = floor(log2 max|x|) over the group, |X| < 2^22, split into balanced digits (see Scheme).
// Every digit is one MMA column; a token owns four. The rounding error is at most 2^-22 max|x|
// per element, 2^-15 max|x| s per group: below 1/60 of that group's share of the 2e-3 sum|x s|
// tolerance. The int32 column sums are exact (each starts at the bits of 1.5 * 2^23, so one
// fp32 subtraction turns it into a float without rounding); the group scale times 2^(e-27) is
// applied once per group in fp32, and the digit weights once per output.
//
// Base-3 storage (b3.cuh) uses the same MMA with u8 weight operands: for a byte q holding n codes,
// F_i = floor(q 3^i / 256) (i = 1 .. n) is the number formed by its first i codes, so
// sum_p x_p c_p = sum_i F_i (x_{i-1} - 3 x_i) (x_n = 0 past the last code): the A operand is
// F_i (0..242, one IMAD per two bytes and a PRMT per four values) and the x side carries the
// combinations x_{i-1} - 3 x_i, built once per call by the prep kernel.
#pragma once

#include "b3.cuh"
#include "bq_internal.cuh"

namespace bq {
namespace mma8 {

constexpr int kColsPerTok = 4;       // MMA columns per token (one per digit of x)
constexpr int kMagic = 0x4B400000;   // bits of 1.5 * 2^23: int n in |n| < 2^22 -> float(bits + n) = 1.5*2^23 + n

// Position of weight k of a group in the MMA operands: quad-thread t (lane % 4) holds register
// rho (0..7) of the A fragment of its two rows; byte b of it is weight k_local(t, rho, b).
// MMA j of the group takes registers 2j (k slots 0..15) and 2j+1 (slots 16..31); the B
// fragment uses the same (t, rho, b) -> k map.
template <int FMT>
__device__ __forceinline__ int k_local(int t, int rho, int b)
{
    if (FMT == BQ_BINARY_G128)
        return 32 * t + 8 * b + rho;                 // bit 8b + rho of word t of the group
    const int h = rho >> 2, r = rho & 3;             // word 2t + h of the group (16 codes)
    const int i = (r == 0) ? 2 * b : (r == 1) ? 8 + 2 * b : (r == 2) ? 2 * b + 1 : 9 + 2 * b;
    return 16 * (2 * t + h) + i;
}

// How x and the weights enter the MMA.
//   kMask (binary): four balanced base-64 digits per token (|d| <= 32); the sign bits enter as
//     b * 2^p with b in {0, 1} (one AND per four weights, p = 5, 6 or 7 by register) and the B
//     byte is d * 2^(7-p) (negated for p = 7, where b * 2^7 is the s8 value -128), so every
//     product is 128 b d; the -64 sum(d) that turns b into 2b - 1 is the MMA's accumulator input,
//     a per-(group, column) value.
//   otherwise (ternary): three balanced base-256 digits and a zero column; the codes enter as
//     {-64, 0, +64} (one PRMT per four codes); the accumulator input is a constant.
//   base-3: three balanced base-256 digits of the level combinations and a zero column; the
//     weights enter as u8 F values; the accumulator input of a column is minus the group's sum of
//     that digit of x (it turns codes c into c - 1), a per-(group, column) value as for binary.
template <int FMT, int CS> struct Scheme {
    static constexpr bool kMask = FMT == BQ_BINARY_G128;
    static constexpr bool kB3 = FMT == BQ_TERNARY_B3_G128;
    static constexpr bool kColFix = kMask || kB3;          // accumulator input per (group, column)
    static constexpr int kCount = kMask ? 4 : 3;
    static constexpr int kBits = kMask ? 6 : 8;
};

// Base-3: byte j and level i (1 .. count(j)) that A-operand slot (t, rho, b) holds. Quad-thread
// t of a group owns five-code bytes 4t .. 4t+3 (registers 0..4 = levels 1..5, byte b = byte 4t+b),
// five-code bytes 16+2t, 17+2t (registers 5, 6, 7: levels 1-2, 3-4, 5, two bytes each) and levels
// 1-2 (t even) or 3-4 (t odd) of four-code byte 24 + t/2 (bytes 2, 3 of register 7).
__host__ __device__ constexpr int b3_slot_byte(int t, int rho, int b)
{
    return rho < 5 ? 4 * t + b : (rho < 7 || b < 2) ? 16 + 2 * t + (b & 1) : 24 + (t >> 1);
}
__host__ __device__ constexpr int b3_slot_level(int t, int rho, int b)
{
    return rho < 5 ? rho + 1 : (rho < 7 || b < 2) ? 2 * (rho - 5) + 1 + (b >> 1) : 2 * (t & 1) + 1 + (b - 2);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// 8 A registers of one row of a base-3 group for quad-thread t: w = its five-code bytes
// 4t..4t+3, h = bytes 16+2t, 17+2t in the low half, tb = its four-code byte, mt = 3^l1 + 2^16 3^l2
// for that byte's two levels. Bytes go to 16-bit lanes, so a multiply by 3^i gives the level-i
// values of two bytes at once in bits 8..15 and 24..31 (q 3^i < 2^16), and a PRMT takes four.
__device__ __forceinline__ void expand_b3(uint32_t w, uint32_t h, uint32_t tb, uint32_t mt, uint32_t *a)
{
    uint32_t pa = prmt(w, 0u, 0x4140u), pb = prmt(w, 0u, 0x4342u), pc = prmt(h, 0u, 0x4140u);
    uint32_t c[6];
    c[0] = pc;
#pragma unroll
    for (int i = 1; i <= 5; i++) {
        pa *= 3u;
        pb *= 3u;
        c[i] = c[i - 1] * 3u;
        a[i - 1] = prmt(pa, pb, 0x7531u);        // level i of bytes 4t .. 4t+3
    }
    a[5] = prmt(c[1], c[2], 0x7531u);
    a[6] = prmt(c[3], c[4], 0x7531u);
    a[7] = prmt(c[5], tb * mt, 0x7531u);
}

// Binary: bit position p that bit (8b + rho) of a word lands on in A register rho, and the
// matching B multiplier 2^(7-p) (-1 for p = 7).
__host__ __device__ constexpr int bin_p(int rho) { return rho == 2 || rho == 5 ? 5 : (rho == 0 || rho == 3 || rho == 6 ? 6 : 7); }
__host__ __device__ constexpr int bin_bmul(int rho) { return bin_p(rho) == 5 ? 4 : (bin_p(rho) == 6 ? 2 : -1); }

// 8 A registers of one binary word (kMask scheme): register rho holds, in byte b, bit 8b + rho
// as b * 2^p (p = bin_p(rho)): registers 5, 6, 7 take bits 5, 6, 7 of each byte straight from
// the word, registers 2, 3, 4 the same bits of the word shifted left by 3, registers 0, 1 by 6.
// Two shifts (multiplies by values held in registers, on the FMA pipe) and eight ANDs (ALU
// pipe) per 32 weights. mk = {8, 64, 0x20202020, 0x40404040, 0x80808080, ...}.
__device__ __forceinline__ void expand_binary_mask(uint32_t w, const uint32_t (&mk)[9], uint32_t *a)
{
    const uint32_t s3 = w * mk[0], s6 = w * mk[1];
    a[0] = s6 & mk[3];
    a[1] = s6 & mk[4];
    a[2] = s3 & mk[2];
    a[3] = s3 & mk[3];
    a[4] = s3 & mk[4];
    a[5] = w & mk[2];
    a[6] = w & mk[3];
    a[7] = w & mk[4];
}

// 4 A registers of one ternary word (16 codes), through a PRMT byte table:
// code 0 -> -64 (0xC0), 1 -> 0, 2 -> +64 (0x40), 3 (invalid) -> 0.
__device__ __forceinline__ void expand_ternary(uint32_t w, uint32_t *a)
{
    const uint32_t table = 0x004000C0u;
    const uint32_t e = w & 0x33333333u;              // codes 0, 2, .., 14 in nibbles 0..7
    const uint32_t o = (w >> 2) & 0x33333333u;       // codes 1, 3, .., 15
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(a[0]) : "r"(table), "r"(e));
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(a[1]) : "r"(table), "r"(e >> 16));
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(a[2]) : "r"(table), "r"(o));
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(a[3]) : "r"(table), "r"(o >> 16));
}

// Expand one group of this thread's two rows straight into the four MMA A operands:
// quad[j] = {row r0 reg 2j, row r1 reg 2j, row r0 reg 2j+1, row r1 reg 2j+1}, the register
// order mma.sync wants, so no copies are needed to form the operand tuples.
template <int FMT, bool MASK>
__device__ __forceinline__ void expand_group(const uint8_t *p0, const uint8_t *p1, const uint32_t (&mul)[9],
                                             uint32_t (&quad)[4][4])
{
    static_assert(MASK == (FMT == BQ_BINARY_G128), "binary weights use the mask expansion");
    uint32_t a0[8], a1[8];
    if (FMT == BQ_BINARY_G128) {
        expand_binary_mask(*reinterpret_cast<const uint32_t *>(p0), mul, a0);
        expand_binary_mask(*reinterpret_cast<const uint32_t *>(p1), mul, a1);
    } else {
        const uint2 w0 = *reinterpret_cast<const uint2 *>(p0);
        const uint2 w1 = *reinterpret_cast<const uint2 *>(p1);
        expand_ternary(w0.x, a0);
        expand_ternary(w0.y, a0 + 4);
        expand_ternary(w1.x, a1);
        expand_ternary(w1.y, a1 + 4);
    }
#pragma unroll
    for (int j = 0; j < 4; j++) {
        quad[j][0] = a0[2 * j];
        quad[j][1] = a1[2 * j];
        quad[j][2] = a0[2 * j + 1];
        quad[j][3] = a1[2 * j + 1];
    }
}

// m16n8k32 with u8 A (base-3 F values) or s8 A, s8 B, s32 accumulators.
template <bool U8>
__device__ __forceinline__ void mma_i8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1)
{
    if (U8)
        asm volatile(
            "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <bool U8>
__device__ __forceinline__ void mma_i8_first(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1, const int (&c)[4])
{
    if (U8)
        asm volatile(
            "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
            : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]), "r"(c[2]), "r"(c[3]));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
            : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]), "r"(c[2]), "r"(c[3]));
}

__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// First MMA of a chain: the accumulator input is a constant quad c (kept in registers).
__device__ __forceinline__ void mma_s8_first(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1, const int (&c)[4])
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]), "r"(c[2]), "r"(c[3]));
}

template <typename T>
__device__ __forceinline__ void store_y(void *y, int yt, int64_t idx, float v)
{
    (void)sizeof(T);
    if (yt == BQ_F32)
        store_out(static_cast<float *>(y) + idx, v);
    else if (yt == BQ_BF16)
        store_out(static_cast<__nv_bfloat16 *>(y) + idx, v);
    else
        store_out(static_cast<__half *>(y) + idx, v);
}

// floor(log2 a) of a finite a > 0, from its bits (subnormals included).
__device__ __forceinline__ int ilog2f(float a)
{
    const uint32_t u = __float_as_uint(a);
    return u >= 0x00800000u ? (int)(u >> 23) - 127 : -118 - (int)__clz(u);
}

// 2^k as a float for k in [-149, 127] (exact; subnormal below -126), 0 below.
__device__ __forceinline__ float pow2f(int k)
{
    if (k >= -126)
        return __uint_as_float((uint32_t)(k + 127) << 23);
    return k >= -149 ? __uint_as_float(1u << (k + 149)) : 0.f;
}

// Digit fragments of token slot m (MMA columns 4m .. 4m+3) in group q, the token's factor
// 2^(e-27) (the weight 2^(kBits d) of digit d is applied once per output) and the accumulator
// inputs of its columns (the bits of 1.5 * 2^23, minus 64 sum(d) over the group for binary),
// written with the layouts [cs][q][half][lane][4] u32, [slot][G] f32 and [cs][q][8] s32.
// One warp builds NT (group, token) items at once, item i = task0 + i * stride of the G * M
// items (q = item / M, m = item % M); the items' reduction chains are independent, so they
// overlap. Lane (t, rho) builds register rho of quad-thread t. Warp-wide maxima and sums are
// single redux.sync instructions. An item past the last is computed on zeros and not stored.
template <int FMT, int CS, typename XT, int NT>
__device__ __forceinline__ void build_items(const XT *__restrict__ x, int M, int64_t K, int G, int task0, int stride,
                                            int lane, uint32_t *__restrict__ frag, float *__restrict__ colf,
                                            int *__restrict__ cfix)
{
    using D = Scheme<FMT, CS>;
    const int t = lane >> 3, rho = lane & 7;
    const int total = G * M;
    float v[NT][4];
#pragma unroll
    for (int i = 0; i < NT; i++) {
        const int item = task0 + i * stride;
        const int q = item / M, m = item % M;
#pragma unroll
        for (int b = 0; b < 4; b++)
            v[i][b] = item < total ? load_x(x + (int64_t)m * K + 128 * q + k_local<FMT>(t, rho, b)) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < NT; i++) {
        const int item = task0 + i * stride;
        const int q = item / M, m = item % M;
        // the group's largest magnitude (non-negative floats order like their bit patterns)
        float amax = fmaxf(fmaxf(fabsf(v[i][0]), fabsf(v[i][1])), fmaxf(fabsf(v[i][2]), fabsf(v[i][3])));
        amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
        // an infinity or NaN in the group: its factor becomes NaN, so the token's outputs are NaN
        const bool bad = __any_sync(0xffffffffu, !(isfinite(v[i][0]) && isfinite(v[i][1]) && isfinite(v[i][2]) &&
                                                   isfinite(v[i][3])));
        if (bad)
            amax = 0.f;                                 // digits of zero; the NaN factor follows
        const int e = amax > 0.f ? ilog2f(amax) : 0;       // amax in [2^e, 2^(e+1))
        // x 2^(21 - e) as two exact power-of-two factors (21 - e can exceed 127 for tiny x)
        const int k = 21 - e;
        const float f1 = pow2f(k < 127 ? k : 127), f2 = pow2f(k > 127 ? k - 127 : 0);
        const int bmul = D::kMask ? bin_bmul(rho) : 1;
        uint32_t dw[4] = {0u, 0u, 0u, 0u};
        int csum[4] = {0, 0, 0, 0};
#pragma unroll
        for (int b = 0; b < 4; b++) {
            int X = amax > 0.f ? __float2int_rn(v[i][b] * f1 * f2) : 0;         // |X| < 2^22
#pragma unroll
            for (int d = 0; d < D::kCount; d++) {
                constexpr int kHalf = 1 << (D::kBits - 1), kMask = (1 << D::kBits) - 1;
                const int dig = ((X + kHalf) & kMask) - kHalf;               // balanced digit
                dw[d] |= ((uint32_t)(dig * bmul) & 0xFFu) << (8 * b);
                csum[d] += dig;
                X = (X - dig) >> D::kBits;                                   // exact
            }
        }
        if (D::kMask) {
#pragma unroll
            for (int d = 0; d < 4; d++)
                csum[d] = __reduce_add_sync(0xffffffffu, csum[d]);
        }
        float fac = amax > 0.f ? pow2f(e - 27) : 0.f;                      // 2^(e-21) / 64
        if (bad)
            fac = __int_as_float(0x7fffffff);
        if (item < total) {
#pragma unroll
            for (int d = 0; d < kColsPerTok; d++) {
                const int c = m * kColsPerTok + d;
                const int cs = c >> 3, ln = 4 * (c & 7) + t;
                frag[(((cs * G + q) * 2 + (rho >> 2)) * 32 + ln) * 4 + (rho & 3)] = d < D::kCount ? dw[d] : 0u;
                if (lane == 0)
                    cfix[(cs * G + q) * 8 + (c & 7)] = kMagic - (D::kMask ? 64 * csum[d] : 0);
            }
            if (lane == 0)
                colf[m * G + q] = fac;
        }
    }
}

// Base-3: the digit fragments, factor and accumulator inputs of one (group, token) item, with the
// layouts of build_items. Lane (t, rho) builds register rho of quad-thread t: slot b holds level i
// of byte j, whose x value is X[k] - 3 X[k+1] (k = first(j) + i - 1, i < count(j)) or X[k] (last
// level), X = round(x 2^(19-e)) with e = floor(log2 max|x|) over the group, so |X| <= 2^20 and
// each value (<= 2^22) has three balanced base-256 digits. The lane also converts positions
// 4 lane .. 4 lane + 3 for the group's maximum and for the sums of the digits of X over the group,
// which the accumulator inputs subtract (codes c become c - 1). Every X of a position is the same
// rounding of the same product wherever it is formed. The column sums stay exact integers: at most
// 128 * (24 * 358 + 2 * 116) + 128 * 128 < 2^21 in magnitude.
template <int CS, typename XT>
__device__ __forceinline__ void build_item_b3(const XT *__restrict__ x, int M, int64_t K, int G, int item, int lane,
                                              uint32_t *__restrict__ frag, float *__restrict__ colf,
                                              int *__restrict__ cfix)
{
    const int t = lane >> 3, rho = lane & 7;
    const bool live = item < G * M;
    const int q = live ? item / M : 0, m = live ? item % M : 0;
    const XT *xg = x + (int64_t)m * K + 128 * q;
    float pv[4], v1[4], v2[4];
    bool two[4];
#pragma unroll
    for (int b = 0; b < 4; b++) {
        const int j = b3_slot_byte(t, rho, b), i = b3_slot_level(t, rho, b);
        const int k1 = b3::first(j) + i - 1;
        two[b] = i < b3::count(j);
        pv[b] = live ? load_x(xg + 4 * lane + b) : 0.f;
        v1[b] = live ? load_x(xg + k1) : 0.f;
        v2[b] = live && two[b] ? load_x(xg + k1 + 1) : 0.f;
    }
    float amax = fmaxf(fmaxf(fabsf(pv[0]), fabsf(pv[1])), fmaxf(fabsf(pv[2]), fabsf(pv[3])));
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    const bool bad = __any_sync(0xffffffffu, !(isfinite(pv[0]) && isfinite(pv[1]) && isfinite(pv[2]) &&
                                               isfinite(pv[3])));
    if (bad)
        amax = 0.f;
    const int e = amax > 0.f ? ilog2f(amax) : 0;
    const int k = 19 - e;
    const float f1 = pow2f(k < 127 ? k : 127), f2 = pow2f(k > 127 ? k - 127 : 0);
    auto to_int = [&](float v) { return amax > 0.f ? __float2int_rn(v * f1 * f2) : 0; };
    uint32_t dw[3] = {0u, 0u, 0u};
    int csum[3] = {0, 0, 0};
#pragma unroll
    for (int b = 0; b < 4; b++) {
        int V = to_int(v1[b]) - (two[b] ? 3 * to_int(v2[b]) : 0);
        int P = to_int(pv[b]);
#pragma unroll
        for (int d = 0; d < 3; d++) {
            const int dig = ((V + 128) & 255) - 128;
            dw[d] |= ((uint32_t)dig & 0xFFu) << (8 * b);
            V = (V - dig) >> 8;
            const int pd = ((P + 128) & 255) - 128;
            csum[d] += pd;
            P = (P - pd) >> 8;
        }
    }
#pragma unroll
    for (int d = 0; d < 3; d++)
        csum[d] = __reduce_add_sync(0xffffffffu, csum[d]);
    float fac = amax > 0.f ? pow2f(e - 19) : 0.f;
    if (bad)
        fac = __int_as_float(0x7fffffff);
    if (live) {
#pragma unroll
        for (int d = 0; d < kColsPerTok; d++) {
            const int c = m * kColsPerTok + d;
            const int cs = c >> 3, ln = 4 * (c & 7) + t;
            frag[(((cs * G + q) * 2 + (rho >> 2)) * 32 + ln) * 4 + (rho & 3)] = d < 3 ? dw[d] : 0u;
            if (lane == 0)
                cfix[(cs * G + q) * 8 + (c & 7)] = kMagic - (d < 3 ? csum[d] : 0);
        }
        if (lane == 0)
            colf[m * G + q] = fac;
    }
}

}  // namespace mma8
}  // namespace bq
