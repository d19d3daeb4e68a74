// embed.cu -- embedding lookup on a packed binary-g128 / ternary-g128 matrix.
//
// out[t][k] = s[id][k/128] * v[id][k], id = ids[t]: the embedding is one of the
// binary layers (model card "prism-ml/Bonsai-27B-mlx-1bit", section "Highlights"; also
// "Model overview", low-bit coverage). The packed row is read once (K/8 bytes binary) and
// the expanded row is written with 16-byte stores; the kernel is bound by the writes.
//
// One warp per token row; a lane expands one packed word at a time (32 binary weights =
// 64 B of bf16, or 16 ternary weights = 32 B).
#include "bq_internal.cuh"

namespace bq {
namespace {

constexpr int kWarps = 8;

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

template <int FMT, typename OT>
__global__ void __launch_bounds__(kWarps * 32)
embed16_kernel(const int32_t *__restrict__ ids, int64_t T, const uint32_t *__restrict__ words,
               const __half *__restrict__ scales, int64_t N, int64_t K, OT *__restrict__ out,
               unsigned int *dev_status)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (t >= T)
        return;
    const int64_t id = ids[t];
    const bool valid = id >= 0 && id < N;
    if (!valid && lane == 0)
        atomicOr(dev_status + kSlotErrBits, kDevErrInvalidId);
    constexpr int KPW = FMT == BQ_BINARY_G128 ? 32 : 16;      // weights per word
    const int64_t W = K / KPW;
    OT *orow = out + t * K;
    for (int64_t w = lane; w < W; w += 32) {
        uint32_t word = 0;
        float s = 0.f;
        if (valid) {
            word = __ldg(words + id * W + w);
            s = __half2float(scales[id * (K / 128) + (w * KPW) / 128]);
        }
        const uint16_t plus = Pack8<OT>::bits(s), minus = plus ^ 0x8000u;
        const uint16_t zero = 0;
        uint32_t o[KPW / 2];
#pragma unroll
        for (int i = 0; i < KPW / 2; i++) {
            uint16_t lo, hi;
            if (FMT == BQ_BINARY_G128) {
                lo = ((word >> (2 * i)) & 1u) ? plus : minus;
                hi = ((word >> (2 * i + 1)) & 1u) ? plus : minus;
            } else {
                uint32_t c0 = (word >> (4 * i)) & 3u, c1 = (word >> (4 * i + 2)) & 3u;
                lo = c0 == 2u ? plus : (c0 == 0u ? minus : zero);
                hi = c1 == 2u ? plus : (c1 == 0u ? minus : zero);
            }
            if (!valid)
                lo = hi = 0;
            o[i] = (uint32_t)lo | ((uint32_t)hi << 16);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(orow + w * KPW);
#pragma unroll
        for (int i = 0; i < KPW / 8; i++)
            dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
    }
}

template <int FMT>
__global__ void __launch_bounds__(kWarps * 32)
embed32_kernel(const int32_t *__restrict__ ids, int64_t T, const uint32_t *__restrict__ words,
               const __half *__restrict__ scales, int64_t N, int64_t K, float *__restrict__ out,
               unsigned int *dev_status)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (t >= T)
        return;
    const int64_t id = ids[t];
    const bool valid = id >= 0 && id < N;
    if (!valid && lane == 0)
        atomicOr(dev_status + kSlotErrBits, kDevErrInvalidId);
    constexpr int KPW = FMT == BQ_BINARY_G128 ? 32 : 16;
    const int64_t W = K / KPW;
    float *orow = out + t * K;
    for (int64_t w = lane; w < W; w += 32) {
        uint32_t word = 0;
        float s = 0.f;
        if (valid) {
            word = __ldg(words + id * W + w);
            s = __half2float(scales[id * (K / 128) + (w * KPW) / 128]);
        }
        float o[KPW];
#pragma unroll
        for (int i = 0; i < KPW; i++) {
            if (FMT == BQ_BINARY_G128) {
                o[i] = ((word >> i) & 1u) ? s : -s;
            } else {
                uint32_t c = (word >> (2 * i)) & 3u;
                o[i] = c == 2u ? s : (c == 0u ? -s : 0.f);
            }
            if (!valid)
                o[i] = 0.f;
        }
        float4 *dst = reinterpret_cast<float4 *>(orow + w * KPW);
#pragma unroll
        for (int i = 0; i < KPW / 4; i++)
            dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
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
            embed16_kernel<BQ_BINARY_G128, __nv_bfloat16><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<__nv_bfloat16 *>(out), dev_status);
        else if (ot == BQ_F16)
            embed16_kernel<BQ_BINARY_G128, __half><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<__half *>(out), dev_status);
        else
            embed32_kernel<BQ_BINARY_G128><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<float *>(out), dev_status);
    } else {
        if (ot == BQ_BF16)
            embed16_kernel<BQ_TERNARY_G128, __nv_bfloat16><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<__nv_bfloat16 *>(out), dev_status);
        else if (ot == BQ_F16)
            embed16_kernel<BQ_TERNARY_G128, __half><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<__half *>(out), dev_status);
        else
            embed32_kernel<BQ_TERNARY_G128><<<blocks, block, 0, s>>>(
                ids, T, words, scales, N, K, static_cast<float *>(out), dev_status);
    }
    return cudaGetLastError();
}

}  // namespace bq
