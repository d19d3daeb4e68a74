// pack.cu -- packing of already-quantised weights into the binary-g128 / ternary-g128
// layouts and the inverse.
//
// Model card "prism-ml/Bonsai-27B-mlx-1bit", section "Weight representation: Binary g128":
// one sign bit per weight, 0 -> -scale, 1 -> +scale. Ternary Bonsai 27B article (wmrh.cn),
// section "局限性与未来发展": ternary values in 2-bit storage.
//
// These kernels are elementwise and bound by device memory: one thread builds one packed
// word from 32 (binary) or 16 (ternary) consecutive int8 values read with 16-byte loads,
// so each warp reads 1 KB (binary) / 512 B (ternary) of q contiguously and writes 128 B
// of words. The base-3 storage (b3.cuh) takes one thread per stored byte, the 4 or 5 codes it
// holds being consecutive q values.
#include "b3.cuh"
#include "bq_internal.cuh"

namespace bq {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t bytes_eq_mask(uint32_t v, uint32_t pattern)
{
    // one bit per byte: bit i set where byte i of v equals the same byte of pattern
    uint32_t d = v ^ pattern;
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < 4; i++)
        r |= (((d >> (8 * i)) & 0xffu) == 0u) << i;
    return r;
}

// Binary: q in {-1, +1}. Word w of row n covers k = 32 w .. 32 w + 31 of that row.
__global__ void pack_binary_kernel(const int8_t *__restrict__ q, int64_t total_words,
                                   uint32_t *__restrict__ words, unsigned int *invalid_count)
{
    int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= total_words)
        return;
    // rows are K/32 words long and q rows K bytes long, so word i reads bytes 32 i .. 32 i + 31
    const uint4 *src = reinterpret_cast<const uint4 *>(q + i * 32);
    uint4 a = __ldg(src), b = __ldg(src + 1);
    uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t word = 0;
    int bad = 0;
#pragma unroll
    for (int j = 0; j < 8; j++) {
        uint32_t plus = bytes_eq_mask(v[j], 0x01010101u);    // +1 -> bit 1
        uint32_t minus = bytes_eq_mask(v[j], 0xffffffffu);   // -1 -> bit 0
        word |= plus << (4 * j);
        bad += 4 - __popc(plus | minus);
    }
    words[i] = word;
    if (bad)
        atomicAdd(invalid_count, (unsigned)bad);
}

// Ternary: q in {-1, 0, +1} -> code q + 1 in 2 bits. Word i covers 16 consecutive q.
__global__ void pack_ternary_kernel(const int8_t *__restrict__ q, int64_t total_words,
                                    uint32_t *__restrict__ words, unsigned int *invalid_count)
{
    int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= total_words)
        return;
    uint4 a = __ldg(reinterpret_cast<const uint4 *>(q + i * 16));
    uint32_t v[4] = {a.x, a.y, a.z, a.w};
    uint32_t word = 0;
    int bad = 0;
#pragma unroll
    for (int j = 0; j < 4; j++) {
#pragma unroll
        for (int b = 0; b < 4; b++) {
            int val = (int)(int8_t)((v[j] >> (8 * b)) & 0xffu);
            uint32_t code = (uint32_t)(val + 1);
            bad += code > 2u;
            word |= (code & 3u) << (2 * (4 * j + b));
        }
    }
    words[i] = word;
    if (bad)
        atomicAdd(invalid_count, (unsigned)bad);
}

__global__ void unpack_kernel(int fmt, const uint32_t *__restrict__ words, int64_t total_words,
                              int8_t *__restrict__ q, unsigned int *invalid_count)
{
    int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= total_words)
        return;
    uint32_t w = __ldg(words + i);
    if (fmt == BQ_BINARY_G128) {
        uint32_t out[8];
#pragma unroll
        for (int j = 0; j < 8; j++) {
            uint32_t r = 0;
#pragma unroll
            for (int b = 0; b < 4; b++) {
                uint32_t bit = (w >> (4 * j + b)) & 1u;
                r |= (bit ? 0x01u : 0xffu) << (8 * b);
            }
            out[j] = r;
        }
        uint4 *dst = reinterpret_cast<uint4 *>(q + i * 32);
        dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
        dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
    } else {
        uint32_t out[4];
        int bad = 0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            uint32_t r = 0;
#pragma unroll
            for (int b = 0; b < 4; b++) {
                uint32_t code = (w >> (2 * (4 * j + b))) & 3u;
                bad += code == 3u;
                uint32_t val = code == 3u ? 0u : (uint32_t)(uint8_t)(int8_t)((int)code - 1);
                r |= val << (8 * b);
            }
            out[j] = r;
        }
        *reinterpret_cast<uint4 *>(q + i * 16) = make_uint4(out[0], out[1], out[2], out[3]);
        if (bad)
            atomicAdd(invalid_count, (unsigned)bad);
    }
}

// Base-3: thread i builds byte j = i % 26 of group (i / 26) % G of row i / (26 G).
__global__ void pack_b3_kernel(const int8_t *__restrict__ q, int64_t N, int64_t K, uint8_t *__restrict__ bytes,
                               unsigned int *invalid_count)
{
    const int64_t G = K / 128;
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= N * G * b3::kGroupBytes)
        return;
    const int j = (int)(i % b3::kGroupBytes);
    const int64_t g = (i / b3::kGroupBytes) % G, n = i / (b3::kGroupBytes * G);
    const int8_t *src = q + n * K + 128 * g + b3::first(j);
    const int cnt = b3::count(j);
    uint32_t v = 0;
    int bad = 0;
    for (int p = 0; p < cnt; p++) {
        const int c = (int)__ldg(src + p) + 1;
        bad += (unsigned)c > 2u;
        v = 3u * v + (unsigned)(c & 3) % 3u;     // first code most significant
    }
    bytes[n * (b3::kGroupBytes * G) + b3::byte_offset(G, g, j)] = (uint8_t)b3::encode(v, cnt);
    if (bad)
        atomicAdd(invalid_count, (unsigned)bad);
}

// Inverse: the codes of one stored byte; a byte the encoding never writes gives q = 0 for its
// codes and is counted.
__global__ void unpack_b3_kernel(const uint8_t *__restrict__ bytes, int64_t N, int64_t K, int8_t *__restrict__ q,
                                 unsigned int *invalid_count)
{
    const int64_t G = K / 128;
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= N * G * b3::kGroupBytes)
        return;
    const int j = (int)(i % b3::kGroupBytes);
    const int64_t g = (i / b3::kGroupBytes) % G, n = i / (b3::kGroupBytes * G);
    const uint32_t byte = __ldg(bytes + n * (b3::kGroupBytes * G) + b3::byte_offset(G, g, j));
    int8_t *dst = q + n * K + 128 * g + b3::first(j);
    const int cnt = b3::count(j);
    bool bad = false;
    for (int p = 0; p < cnt; p++) {
        const int c = b3::code(byte, cnt, p);
        bad |= c < 0;
        dst[p] = (int8_t)(c < 0 ? 0 : c - 1);
    }
    if (bad)
        atomicAdd(invalid_count, 1u);
}

inline unsigned blocks_for(int64_t n) { return (unsigned)((n + kThreads - 1) / kThreads); }

}  // namespace

cudaError_t launch_pack_binary(const int8_t *q, int64_t N, int64_t K, uint32_t *words,
                               unsigned int *invalid_count, cudaStream_t s)
{
    int64_t total = N * (K / 32);
    pack_binary_kernel<<<blocks_for(total), kThreads, 0, s>>>(q, total, words, invalid_count);
    return cudaGetLastError();
}

cudaError_t launch_pack_ternary(const int8_t *q, int64_t N, int64_t K, uint32_t *words,
                                unsigned int *invalid_count, cudaStream_t s)
{
    int64_t total = N * (K / 16);
    pack_ternary_kernel<<<blocks_for(total), kThreads, 0, s>>>(q, total, words, invalid_count);
    return cudaGetLastError();
}

cudaError_t launch_pack_b3(const int8_t *q, int64_t N, int64_t K, uint8_t *bytes, unsigned int *invalid_count,
                           cudaStream_t s)
{
    const int64_t total = N * (K / 128) * b3::kGroupBytes;
    pack_b3_kernel<<<blocks_for(total), kThreads, 0, s>>>(q, N, K, bytes, invalid_count);
    return cudaGetLastError();
}

cudaError_t launch_unpack(int fmt, const uint32_t *words, int64_t N, int64_t K, int8_t *q,
                          unsigned int *invalid_count, cudaStream_t s)
{
    if (fmt == BQ_TERNARY_B3_G128) {
        const int64_t total = N * (K / 128) * b3::kGroupBytes;
        unpack_b3_kernel<<<blocks_for(total), kThreads, 0, s>>>(reinterpret_cast<const uint8_t *>(words), N, K, q,
                                                                invalid_count);
        return cudaGetLastError();
    }
    int64_t total = N * (fmt == BQ_BINARY_G128 ? K / 32 : K / 16);
    unpack_kernel<<<blocks_for(total), kThreads, 0, s>>>(fmt, words, total, q, invalid_count);
    return cudaGetLastError();
}

}  // namespace bq
