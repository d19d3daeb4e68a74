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
// Binary: the matrix is read as one run of N K / 128 groups (group f starts at element 128 f);
// a warp takes pairs of groups with one 16-byte load per lane and pair (8 weights: positions
// 8 l .. 8 l + 7 of the pair), builds the 8 sign bits of its weights, ORs four lanes' bytes into a
// packed word and sums |w| over the 16 lanes of its group.
// Ternary: one warp per group; lane l holds positions l, 32 + l, 64 + l, 96 + l. Ternary sorts the 128 magnitudes (their binary32 bits,
// which order like the values) with a bitonic network across the warp, scans them, and takes the
// arg-max of the scores with a warp reduction. Equal magnitudes are adjacent in any sorted order,
// so the prefix sums and the chosen j do not depend on how ties were ordered; the tie rule (lower
// position first) is applied afterwards: every |w| above the j-th largest is in, and of those equal
// to it the lowest positions fill the rest (ballots and prefix counts). The codes go through a
// 128-byte array per warp in shared memory, from which lanes build the 2-bit words or the base-3
// bytes.
#include "b3.cuh"
#include "bq_internal.cuh"

namespace bq {
namespace {

constexpr int kWarps = 8;

template <typename WT> __device__ __forceinline__ float wload(const WT *p);
template <> __device__ __forceinline__ float wload(const float *p) { return __ldg(p); }
template <> __device__ __forceinline__ float wload(const __half *p) { return __half2float(__ldg(p)); }
template <> __device__ __forceinline__ float wload(const __nv_bfloat16 *p) { return __bfloat162float(__ldg(p)); }

// Descending bitonic sort of the warp's 128 keys, key[r] being element 32 r + lane.
__device__ __forceinline__ void sort128_desc(uint32_t (&key)[4], int lane)
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
                        const uint32_t a = key[r], b = key[r | rs];
                        const uint32_t hi = a > b ? a : b, lo = a > b ? b : a;
                        key[r] = desc ? hi : lo;
                        key[r | rs] = desc ? lo : hi;
                    }
                }
            } else {
#pragma unroll
                for (int r = 0; r < 4; r++) {
                    const int e = 32 * r + lane;
                    const uint32_t other = __shfl_xor_sync(0xffffffffu, key[r], stride);
                    // the lower element keeps the larger key in a descending run
                    const bool keep_max = ((e & size) == 0) == ((e & stride) == 0);
                    key[r] = keep_max ? max(key[r], other) : min(key[r], other);
                }
            }
        }
    }
}

// Eight consecutive weights as floats (one 16-byte load for 2-byte types, two for fp32).
template <typename WT> __device__ __forceinline__ void load8(const WT *p, float (&v)[8]);
template <> __device__ __forceinline__ void load8(const float *p, float (&v)[8])
{
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p)), b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <> __device__ __forceinline__ void load8(const __half *p, float (&v)[8])
{
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        v[2 * i] = __half2float(__ushort_as_half((unsigned short)(w[i] & 0xFFFFu)));
        v[2 * i + 1] = __half2float(__ushort_as_half((unsigned short)(w[i] >> 16)));
    }
}
template <> __device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8])
{
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Binary fit of kPairs pairs of groups per warp (flat group indices 2 p, 2 p + 1 for each pair p):
// lane l takes group 2 p + l / 16, weights 8 (l % 16) .. + 7 of it, i.e. bits 8 (l % 4) .. + 7 of
// word (l % 16) / 4. All the warp's loads are issued before any is used, so that enough bytes are
// in flight per SM to keep HBM busy.
constexpr int kPairs = 4;

template <typename WT>
__global__ void __launch_bounds__(kWarps * 32)
quantize_binary_kernel(const WT *__restrict__ w, int64_t groups, uint32_t *__restrict__ words,
                       uint16_t *__restrict__ scales)
{
    const int lane = threadIdx.x & 31, sub = lane & 15;
    const int64_t pair0 = ((int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5)) * kPairs;
    if (2 * pair0 >= groups)
        return;                                        // warp-uniform
    float v[kPairs][8];
#pragma unroll
    for (int u = 0; u < kPairs; u++) {
        const int64_t f = 2 * (pair0 + u) + (lane >> 4);
#pragma unroll
        for (int i = 0; i < 8; i++)
            v[u][i] = 0.f;
        if (f < groups)                                // past the last group: nothing to load
            load8(w + f * 128 + 8 * sub, v[u]);
    }
#pragma unroll
    for (int u = 0; u < kPairs; u++) {
        const int64_t f = 2 * (pair0 + u) + (lane >> 4);
        uint32_t bits = 0;
        double a = 0.0;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            bits |= (v[u][i] >= 0.f ? 1u : 0u) << i;   // 1 -> +s
            a += fabs((double)v[u][i]);
        }
        uint32_t word = bits << (8 * (sub & 3));
        word |= __shfl_xor_sync(0xffffffffu, word, 1);
        word |= __shfl_xor_sync(0xffffffffu, word, 2);
#pragma unroll
        for (int m = 1; m < 16; m <<= 1)
            a += __shfl_xor_sync(0xffffffffu, a, m);
        if (f < groups && (sub & 3) == 0)
            words[f * 4 + (sub >> 2)] = word;
        if (f < groups && sub == 0)
            scales[f] = __half_as_ushort(__double2half(a / 128.0));
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

    static_assert(FMT != BQ_BINARY_G128, "binary groups use quantize_binary_kernel");
    // ternary: sort the magnitudes descending
    uint32_t key[4], mag[4];
#pragma unroll
    for (int r = 0; r < 4; r++)
        key[r] = mag[r] = __float_as_uint(v[r]) & 0x7FFFFFFFu;
    sort128_desc(key, lane);
    // prefix sums of the sorted magnitudes (element 32 r + lane), scores, arg-max
    double base = 0.0, best = 0.0, best_sum = 0.0;
    int best_j = 0;
#pragma unroll
    for (int r = 0; r < 4; r++) {
        double x = (double)__uint_as_float(key[r]);
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
    // the support: every magnitude above the best_j-th largest (mstar), then the lowest
    // positions among those equal to it until best_j are in
    uint32_t mstar = 0xFFFFFFFFu;
    if (best_j > 0) {
        const int e = best_j - 1;                  // warp-uniform
        const uint32_t kr = (e >> 5) == 0 ? key[0] : (e >> 5) == 1 ? key[1] : (e >> 5) == 2 ? key[2] : key[3];
        mstar = __shfl_sync(0xffffffffu, kr, e & 31);
    }
    int need = best_j;
#pragma unroll
    for (int r = 0; r < 4; r++)
        need -= __popc(__ballot_sync(0xffffffffu, mag[r] > mstar));
    const uint32_t below = (1u << lane) - 1u;
    int taken = 0;                                 // equal magnitudes at lower positions so far
#pragma unroll
    for (int r = 0; r < 4; r++) {
        const int pos = 32 * r + lane;
        const uint32_t eq = __ballot_sync(0xffffffffu, mag[r] == mstar);
        const bool in = best_j > 0 && (mag[r] > mstar || (mag[r] == mstar && taken + __popc(eq & below) < need));
        taken += __popc(eq);
        codes_s[warp][pos] = (int8_t)((in ? (v[r] >= 0.f ? 1 : -1) : 0) + 1);
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

cudaError_t launch_binary(const void *w, int wt, int64_t N, int64_t K, void *packed, uint16_t *scales, cudaStream_t s)
{
    const int64_t groups = N * (K / 128), pairs = (groups + 1) / 2;
    const unsigned blocks = (unsigned)((pairs + kWarps * kPairs - 1) / (kWarps * kPairs));
    uint32_t *words = static_cast<uint32_t *>(packed);
    if (wt == BQ_F32)
        quantize_binary_kernel<float><<<blocks, kWarps * 32, 0, s>>>(static_cast<const float *>(w), groups, words, scales);
    else if (wt == BQ_BF16)
        quantize_binary_kernel<__nv_bfloat16><<<blocks, kWarps * 32, 0, s>>>(static_cast<const __nv_bfloat16 *>(w),
                                                                             groups, words, scales);
    else
        quantize_binary_kernel<__half><<<blocks, kWarps * 32, 0, s>>>(static_cast<const __half *>(w), groups, words,
                                                                      scales);
    return cudaGetLastError();
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
        return launch_binary(w, wt, N, K, packed, scales, s);
    if (fmt == BQ_TERNARY_G128)
        return launch_q<BQ_TERNARY_G128>(w, wt, N, K, packed, scales, s);
    return launch_q<BQ_TERNARY_B3_G128>(w, wt, N, K, packed, scales, s);
}

}  // namespace bq
