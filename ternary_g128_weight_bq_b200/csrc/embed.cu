// embed.cu -- embedding lookup on a packed binary-g128 / ternary-g128 matrix.
//
// out[t][k] = s[id][k/128] * v[id][k], id = ids[t]: the embedding is one of the
// binary layers (model card "prism-ml/Bonsai-27B-mlx-1bit", section "Highlights"; also
// "Model overview", low-bit coverage). The packed row is read once (K/8 bytes binary) and
// the expanded row is written with 16-byte stores; the kernel is bound by the writes.
//
// One warp per token row. The row is cut into 8-weight chunks (one byte of a binary word,
// half of a ternary word); lane l takes chunks l, l + 32, ..., so each warp store covers one
// contiguous 512-byte (bf16/fp16) or 1 KB (fp32) span of the output row. The packed bytes of
// four chunks are loaded before any is expanded, so their loads overlap. Base-3 rows (b3.cuh) are
// turned into the 2-bit codes of a chunk on load (its 8 codes sit in 2 or 3 bytes) and expanded
// like ternary ones.
#include <type_traits>

#include "b3.cuh"
#include "bq_internal.cuh"

namespace bq {
namespace {

constexpr int kWarps = 8;
constexpr int kBatch = 4;             // chunks per lane whose loads are in flight together

template <typename OT> struct Pack8;
template <> struct Pack8<__nv_bfloat16> {
    // +-s and 0 in bf16: RNE of the fp16 scale, sign applied after rounding (exact)
    static __device__ __forceinline__ uint16_t bits(float v) {
        return __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
};
template <> struct Pack8<__half> {
    static __device__ __forceinline__ uint16_t bits(float v) { return __half_as_ushort(__float2half_rn(v)); }
};
template <> struct Pack8<float> {
    static __device__ __forceinline__ uint32_t bits(float v) { return __float_as_uint(v); }
};

// The 8 codes of chunk q of a packed row (binary: byte q % 4 of word q / 4; ternary: 16-bit
// half q % 2 of word q / 2), as the low 8 or 16 bits.
template <int FMT>
__device__ __forceinline__ uint32_t load_chunk(const uint32_t *__restrict__ row, int64_t q, int64_t G)
{
    if (FMT == BQ_BINARY_G128)
        return (__ldg(row + (q >> 2)) >> (8 * (q & 3))) & 0xFFu;
    if (FMT == BQ_TERNARY_G128)
        return (__ldg(row + (q >> 1)) >> (16 * (q & 1))) & 0xFFFFu;
    // base-3: positions 8 (q % 16) .. + 7 of group q / 16; a byte the encoding never writes
    // gives code 1 (a zero weight)
    const uint8_t *rb = reinterpret_cast<const uint8_t *>(row);
    const int64_t g = q >> 4;
    const int kk0 = 8 * (int)(q & 15);
    uint32_t codes = 0, byte = 0;
    int jprev = -1;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const int kk = kk0 + i, j = b3::byte_of(kk);
        if (j != jprev) {
            byte = __ldg(rb + b3::byte_offset(G, g, j));
            jprev = j;
        }
        const int c = b3::code(byte, b3::count(j), kk - b3::first(j));
        codes |= (uint32_t)(c < 0 ? 1 : c) << (2 * i);
    }
    return codes;
}

// Value of weight i (0..7) of a chunk: +s / -s (binary bit 1 / 0), +s / 0 / -s (ternary code
// 2 / 1 / 0; code 3, never written by the pack calls, gives 0), as output-type bits.
template <int FMT, typename B>
__device__ __forceinline__ B weight_bits(uint32_t codes, int i, B plus, B minus)
{
    if (FMT == BQ_BINARY_G128)
        return ((codes >> i) & 1u) ? plus : minus;
    const uint32_t c = (codes >> (2 * i)) & 3u;
    return c == 2u ? plus : (c == 0u ? minus : (B)0);
}

template <int FMT, typename OT>
__global__ void __launch_bounds__(kWarps * 32)
embed_kernel(const int32_t *__restrict__ ids, int64_t T, const uint32_t *__restrict__ words,
             const __half *__restrict__ scales, int64_t N, int64_t K, OT *__restrict__ out,
             unsigned int *dev_status)
{
    using B = typename std::conditional<sizeof(OT) == 4, uint32_t, uint16_t>::type;
    constexpr B kSign = sizeof(OT) == 4 ? (B)0x80000000u : (B)0x8000u;
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (t >= T)
        return;
    const int64_t id = ids[t];
    const bool valid = id >= 0 && id < N;
    if (!valid && lane == 0)
        atomicOr(dev_status + kSlotErrBits, kDevErrInvalidId);
    constexpr int KPW = FMT == BQ_BINARY_G128 ? 32 : 16;      // weights per word (2-bit or binary)
    const int64_t G = K / 128;
    const uint32_t *row = FMT == BQ_TERNARY_B3_G128
        ? reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint8_t *>(words) +
                                             (valid ? id : 0) * (b3::kGroupBytes * G))
        : words + (valid ? id : 0) * (K / KPW);
    const __half *srow = scales + (valid ? id : 0) * (K / 128);
    OT *orow = out + t * K;
    const int64_t nq = K / 8;                                  // 8-weight chunks in the row
    for (int64_t q0 = lane; q0 < nq; q0 += 32 * kBatch) {
        uint32_t codes[kBatch];
        float s[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; j++) {
            const int64_t q = q0 + 32 * j;
            codes[j] = 0u;
            s[j] = 0.f;
            if (valid && q < nq) {
                codes[j] = load_chunk<FMT>(row, q, G);
                s[j] = __half2float(srow[q >> 4]);             // 16 chunks per group of 128
            }
        }
#pragma unroll
        for (int j = 0; j < kBatch; j++) {
            const int64_t q = q0 + 32 * j;
            if (q >= nq)
                break;
            const B plus = valid ? (B)Pack8<OT>::bits(s[j]) : (B)0;
            const B minus = valid ? (B)(plus ^ kSign) : (B)0;
            B o[8];
#pragma unroll
            for (int i = 0; i < 8; i++)
                o[i] = weight_bits<FMT, B>(codes[j], i, plus, minus);
            if (sizeof(OT) == 2) {
                uint4 v;
                v.x = (uint32_t)o[0] | ((uint32_t)o[1] << 16);
                v.y = (uint32_t)o[2] | ((uint32_t)o[3] << 16);
                v.z = (uint32_t)o[4] | ((uint32_t)o[5] << 16);
                v.w = (uint32_t)o[6] | ((uint32_t)o[7] << 16);
                *reinterpret_cast<uint4 *>(orow + 8 * q) = v;
            } else {
                uint4 *d = reinterpret_cast<uint4 *>(orow + 8 * q);
                d[0] = make_uint4((uint32_t)o[0], (uint32_t)o[1], (uint32_t)o[2], (uint32_t)o[3]);
                d[1] = make_uint4((uint32_t)o[4], (uint32_t)o[5], (uint32_t)o[6], (uint32_t)o[7]);
            }
        }
    }
}

}  // namespace

cudaError_t launch_embed(int fmt, const int32_t *ids, int64_t T, const uint32_t *words,
                         const __half *scales, int64_t N, int64_t K, void *out, int ot,
                         unsigned int *dev_status, cudaStream_t s)
{
    unsigned blocks = (unsigned)((T + kWarps - 1) / kWarps);
    dim3 block(kWarps * 32);
    if (fmt == BQ_BINARY_G128) {
        if (ot == BQ_BF16)
            embed_kernel<BQ_BINARY_G128, __nv_bfloat16><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<__nv_bfloat16 *>(out), dev_status);
        else if (ot == BQ_F16)
            embed_kernel<BQ_BINARY_G128, __half><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<__half *>(out), dev_status);
        else
            embed_kernel<BQ_BINARY_G128, float><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<float *>(out), dev_status);
    } else if (fmt == BQ_TERNARY_G128) {
        if (ot == BQ_BF16)
            embed_kernel<BQ_TERNARY_G128, __nv_bfloat16><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<__nv_bfloat16 *>(out), dev_status);
        else if (ot == BQ_F16)
            embed_kernel<BQ_TERNARY_G128, __half><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<__half *>(out), dev_status);
        else
            embed_kernel<BQ_TERNARY_G128, float><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<float *>(out), dev_status);
    } else {
        if (ot == BQ_BF16)
            embed_kernel<BQ_TERNARY_B3_G128, __nv_bfloat16><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<__nv_bfloat16 *>(out), dev_status);
        else if (ot == BQ_F16)
            embed_kernel<BQ_TERNARY_B3_G128, __half><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<__half *>(out), dev_status);
        else
            embed_kernel<BQ_TERNARY_B3_G128, float><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<float *>(out), dev_status);
    }
    return cudaGetLastError();
}

}  // namespace bq
