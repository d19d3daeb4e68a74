// quantize.cu -- dense weights to the packed g128 formats: the least-squares fit of every group of
// 128 weights, then the format's packing.
//
// The pages name the formats (model card "prism-ml/Bonsai-27B-mlx-1bit", section "Weight
// representation: Binary g128"; Ternary Bonsai 27B article, wmrh.cn) but not how q and s are
// obtained, so this library takes the least-squares fit of each group of 128 weights w:
//   binary:  q = +1 where w >= 0, else -1, and s = mean |w| (the best scale for those signs);
//   ternary: q in {-1, 0, +1} and s minimising sum (w - s q)^2: a support of j weights leaves
//            sum w^2 - (sum_support |w|)^2 / j, so the support is the j largest |w| (equal |w|:
//            lower position first) with j maximising (sum |w|)^2 / j (the smallest such j; no
//            support for a group of zeros), q their signs and s their mean |w|.
// s is rounded to fp16 (nearest even). Sums and scores are taken in fp64, which holds the sum of
// 128 binary32 magnitudes exactly unless their exponents span more than about 29 binades, so the
// choice of j does not depend on the order of the additions.
//
// One warp per group; lane l holds positions l, 32 + l, 64 + l, 96 + l. Binary signs are four
// ballots (the packed words themselves). Ternary sorts 128 keys (|w| bits, then the position)
// with a bitonic network across the warp, scans the sorted magnitudes, and takes the arg-max of
// the scores with a warp reduction; the codes go through a 128-byte array per warp in shared
// memory, from which lanes build the 2-bit words or the base-3 bytes.
#include "b3.cuh"
#include "bq_internal.cuh"

namespace bq {
namespace {

constexpr int kWarps = 8;

template <typename WT> __device__ __forceinline__ float wload(const WT *p);
template <> __device__ __forceinline__ float wload(const float *p) { return __ldg(p); }
template <> __device__ __forceinline__ float wload(const __half *p) { return __half2float(__ldg(p)); }
template <> __device__ __forceinline__ float wload(const __nv_bfloat16 *p) { return __bfloat162float(__ldg(p)); }

__device__ __forceinline__ unsigned long long shfl_xor64(unsigned long long v, int m)
{
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
    return ((unsigned long long)hi << 32) | lo;
}

__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

// Descending bitonic sort of the warp's 128 keys, key[r] being element 32 r + lane.
__device__ __forceinline__ void sort128_desc(unsigned long long (&key)[4], int lane)
{
#pragma unroll
    for (int size = 2; size <= 128; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride >= 1; stride >>= 1) {
            if (stride >= 32) {
                const int rs = stride >> 5;
#pragma unroll
                for (int r = 0; r < 4; r++) {
                    if ((r & rs) == 0) {
                        const int e = 32 * r + lane;
                        const bool desc = (e & size) == 0;
                        const unsigned long long a = key[r], b = key[r | rs];
                        const bool swap = desc ? a < b : a > b;
                        key[r] = swap ? b : a;
                        key[r | rs] = swap ? a : b;
                    }
                }
            } else {
#pragma unroll
                for (int r = 0; r < 4; r++) {
                    const int e = 32 * r + lane;
                    const unsigned long long other = shfl_xor64(key[r], stride);
                    const bool desc = (e & size) == 0;
                    const bool lower = (e & stride) == 0;
                    // the lower element keeps the larger key in a descending run
                    const bool keep_max = desc == lower;
                    key[r] = keep_max ? (key[r] > other ? key[r] : other) : (key[r] < other ? key[r] : other);
                }
            }
        }
    }
}

template <int FMT, typename WT>
__global__ void __launch_bounds__(kWarps * 32)
quantize_kernel(const WT *__restrict__ w, int64_t N, int64_t K, void *__restrict__ packed, uint16_t *__restrict__ scales)
{
    __shared__ int8_t codes_s[kWarps][128];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t G = K / 128;
    const int64_t item = (int64_t)blockIdx.x * kWarps + warp;       // (row, group)
    if (item >= N * G)
        return;
    const int64_t n = item / G, g = item % G;
    const WT *wg = w + n * K + 128 * g;
    float v[4];
#pragma unroll
    for (int r = 0; r < 4; r++)
        v[r] = wload(wg + 32 * r + lane);

    if constexpr (FMT == BQ_BINARY_G128) {
        uint32_t *words = static_cast<uint32_t *>(packed) + n * (K / 32) + 4 * g;
        double a = 0.0;
#pragma unroll
        for (int r = 0; r < 4; r++) {
            const uint32_t bits = __ballot_sync(0xffffffffu, v[r] >= 0.f);     // 1 -> +s
            if (lane == r)
                words[r] = bits;
            a += fabs((double)v[r]);
        }
        const double sum = warp_sum(a);
        if (lane == 0)
            scales[n * G + g] = __half_as_ushort(__double2half(sum / 128.0));
    } else {
        // ternary: sort (|w|, position) descending
        unsigned long long key[4];
#pragma unroll
        for (int r = 0; r < 4; r++)
            key[r] = ((unsigned long long)(__float_as_uint(v[r]) & 0x7FFFFFFFu) << 32) |
                     (0xFFFFFFFFu - (uint32_t)(32 * r + lane));
        sort128_desc(key, lane);
        // prefix sums of the sorted magnitudes (element 32 r + lane), scores, arg-max
        double base = 0.0, best = 0.0, best_sum = 0.0;
        int best_j = 0;
#pragma unroll
        for (int r = 0; r < 4; r++) {
            double x = (double)__uint_as_float((uint32_t)(key[r] >> 32));
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const double o = __shfl_up_sync(0xffffffffu, x, d);
                if (lane >= d)
                    x += o;
            }
            const double prefix = base + x;
            const int j = 32 * r + lane + 1;
            const double score = prefix * prefix / j;
            if (score > best) {                       // j grows with r: the first maximum per lane
                best = score;
                best_j = j;
                best_sum = prefix;
            }
            base = __shfl_sync(0xffffffffu, prefix, 31);
        }
        // warp arg-max: largest score, then smallest j
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
            const double ob = __shfl_xor_sync(0xffffffffu, best, m);
            const int oj = __shfl_xor_sync(0xffffffffu, best_j, m);
            const double os = __shfl_xor_sync(0xffffffffu, best_sum, m);
            if (ob > best || (ob == best && oj < best_j && ob > 0.0)) {
                best = ob;
                best_j = oj;
                best_sum = os;
            }
        }
        // the support is the best_j largest keys: those >= the key at sorted position best_j - 1
        unsigned long long thr = ~0ull;
        if (best_j > 0) {
            const int e = best_j - 1;
            const unsigned long long kr = key[e >> 5];
            thr = __shfl_sync(0xffffffffu, kr, e & 31);
        }
        // (every lane took part in the shuffle above; the key of register e >> 5 of lane e & 31)
#pragma unroll
        for (int r = 0; r < 4; r++) {
            const int pos = 32 * r + lane;
            const unsigned long long mine = ((unsigned long long)(__float_as_uint(v[r]) & 0x7FFFFFFFu) << 32) |
                                            (0xFFFFFFFFu - (uint32_t)pos);
            const int q = best_j > 0 && mine >= thr ? (v[r] >= 0.f ? 1 : -1) : 0;
            codes_s[warp][pos] = (int8_t)(q + 1);
        }
        __syncwarp();
        if (lane == 0)
            scales[n * G + g] = __half_as_ushort(__double2half(best_j ? best_sum / best_j : 0.0));
        const int8_t *c = codes_s[warp];
        if (FMT == BQ_TERNARY_G128) {
            if (lane < 8) {                            // 8 words of 16 codes
                uint32_t word = 0;
#pragma unroll
                for (int i = 0; i < 16; i++)
                    word |= (uint32_t)c[16 * lane + i] << (2 * i);
                static_cast<uint32_t *>(packed)[n * (K / 16) + 8 * g + lane] = word;
            }
        } else {
            if (lane < b3::kGroupBytes) {
                const int cnt = b3::count(lane), k0 = b3::first(lane);
                uint32_t val = 0;
                for (int p = 0; p < cnt; p++)
                    val = 3u * val + (uint32_t)c[k0 + p];
                static_cast<uint8_t *>(packed)[n * (b3::kGroupBytes * G) + b3::byte_offset(G, g, lane)] =
                    (uint8_t)b3::encode(val, cnt);
            }
        }
    }
}

template <int FMT>
cudaError_t launch_q(const void *w, int wt, int64_t N, int64_t K, void *packed, uint16_t *scales, cudaStream_t s)
{
    const int64_t items = N * (K / 128);
    const unsigned blocks = (unsigned)((items + kWarps - 1) / kWarps);
    if (wt == BQ_F32)
        quantize_kernel<FMT, float><<<blocks, kWarps * 32, 0, s>>>(static_cast<const float *>(w), N, K, packed, scales);
    else if (wt == BQ_BF16)
        quantize_kernel<FMT, __nv_bfloat16><<<blocks, kWarps * 32, 0, s>>>(static_cast<const __nv_bfloat16 *>(w), N,
                                                                           K, packed, scales);
    else
        quantize_kernel<FMT, __half><<<blocks, kWarps * 32, 0, s>>>(static_cast<const __half *>(w), N, K, packed,
                                                                    scales);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(int fmt, const void *w, int wt, int64_t N, int64_t K, void *packed, uint16_t *scales,
                            cudaStream_t s)
{
    if (fmt == BQ_BINARY_G128)
        return launch_q<BQ_BINARY_G128>(w, wt, N, K, packed, scales, s);
    if (fmt == BQ_TERNARY_G128)
        return launch_q<BQ_TERNARY_G128>(w, wt, N, K, packed, scales, s);
    return launch_q<BQ_TERNARY_B3_G128>(w, wt, N, K, packed, scales, s);
}

}  // namespace bq
