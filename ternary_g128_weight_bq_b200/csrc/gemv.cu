// gemv.cu -- decode GEMV on packed binary-g128 / ternary-g128 weights (2-bit or base-3
// storage), M <= 8 token rows.
//
// y[m][n] = sum_g s[n][g] * sum_{k in g} v[n][k] * x[m][k],  v = 2b - 1 (binary) or c - 1
// (ternary). Model card "prism-ml/Bonsai-27B-mlx-1bit", sections "Weight representation:
// Binary g128" and "CUDA (NVIDIA GPUs)"; the batch-1 decode (tg128) workload of section
// "Cross-platform throughput".
//
// SIMT kernel: each sign bit is applied to x by select-and-add (never a multiply), each
// group is reduced in fp32, the group scale is applied once per group, and the lanes that
// share a row are combined with warp shuffles.
//   * 8 lanes per row, 4 rows per warp: the 8 lanes of a row read 8 consecutive 16-byte
//     groups (128 B contiguous), so a warp's load touches 4 full 128-byte lines.
//   * the activations are staged once per block into shared memory as fp32 when they fit
//     (M*K*4 <= 200 KB), else read from global memory (L1/L2-resident).
// This kernel serves the shapes the tensor-core kernel (gemv_rows.cu) does not take: K not a
// multiple of 1024, or digit fragments too large for shared memory.
#include "b3.cuh"
#include "bq_internal.cuh"

namespace bq {
namespace {

constexpr int kSimtThreads = 256;        // 8 warps
constexpr int kRowsPerBlock = 32;        // 4 rows per warp
constexpr int kSimtMaxSmem = 200 * 1024;

template <typename XT>
__device__ __forceinline__ float xval(const XT *p) { return load_x(p); }

// x is read from shared memory (fp32, when M*K*4 fits) or straight from global memory.
template <bool SMEM_X, typename XT>
struct XSrc {
    const float *s;
    const XT *g;
    __device__ __forceinline__ float operator[](int64_t i) const { return SMEM_X ? s[i] : xval(g + i); }
};

template <int FMT, int M, typename XT, bool SMEM_X>
__global__ void __launch_bounds__(kSimtThreads)
gemv_simt_kernel(const XT *__restrict__ x, int64_t K, const uint32_t *__restrict__ words,
                 const __half *__restrict__ scales, int64_t N, void *__restrict__ y, int yt)
{
    extern __shared__ float xs_raw[];   // [M][K] fp32 when SMEM_X
    if (SMEM_X) {
        for (int64_t i = threadIdx.x; i < (int64_t)M * K; i += kSimtThreads)
            xs_raw[i] = xval(x + i);
        __syncthreads();
    }
    const XSrc<SMEM_X, XT> xs{xs_raw, x};

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane >> 3, j = lane & 7;
    const int64_t n = (int64_t)blockIdx.x * kRowsPerBlock + warp * 4 + sub;
    const int64_t G = K / 128;
    float acc[M];
#pragma unroll
    for (int m = 0; m < M; m++)
        acc[m] = 0.f;

    if (n < N) {
        constexpr int WPG = FMT == BQ_BINARY_G128 ? 4 : 8;     // words per group (not base-3)
        const uint32_t *wrow = words + n * G * WPG;
        const uint8_t *brow = reinterpret_cast<const uint8_t *>(words) + n * G * b3::kGroupBytes;
        for (int64_t g = j; g < G; g += 8) {
            uint32_t w[WPG];
            if (FMT != BQ_TERNARY_B3_G128) {
#pragma unroll
                for (int i = 0; i < WPG; i += 4) {
                    uint4 v = __ldg(reinterpret_cast<const uint4 *>(wrow + g * WPG + i));
                    w[i] = v.x; w[i + 1] = v.y; w[i + 2] = v.z; w[i + 3] = v.w;
                }
            }
            const float s = __half2float(scales[n * G + g]);
            float part[M];
#pragma unroll
            for (int m = 0; m < M; m++)
                part[m] = 0.f;
            const int64_t xg = g * 128;
            if (FMT == BQ_BINARY_G128) {
#pragma unroll
                for (int i = 0; i < 4; i++) {
#pragma unroll 8
                    for (int b = 0; b < 32; b++) {
                        const bool on = (w[i] >> b) & 1u;      // 1 -> +x, 0 -> -x
#pragma unroll
                        for (int m = 0; m < M; m++) {
                            float xv = xs[xg + m * K + i * 32 + b];
                            part[m] += on ? xv : -xv;
                        }
                    }
                }
            } else if (FMT == BQ_TERNARY_B3_G128) {
                // byte jb holds codes first(jb) .. first(jb) + count(jb) - 1 of the group;
                // code p is F_{p+1} - 3 F_p with F_i = floor(q 3^i / 256)
                for (int jb = 0; jb < b3::kGroupBytes; jb++) {
                    const uint32_t qb = __ldg(brow + b3::byte_offset(G, g, jb));
                    const int cnt = b3::count(jb), k0 = b3::first(jb);
                    uint32_t fprev = 0;
#pragma unroll
                    for (int p = 0; p < 5; p++) {
                        if (p < cnt) {
                            const uint32_t f = (qb * b3::pow3(p + 1)) >> 8;
                            const uint32_t c = f - 3u * fprev;
                            fprev = f;
#pragma unroll
                            for (int m = 0; m < M; m++) {
                                float xv = xs[xg + m * K + k0 + p];
                                part[m] += c == 2u ? xv : (c == 0u ? -xv : 0.f * xv);
                            }
                        }
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; i++) {
#pragma unroll 4
                    for (int b = 0; b < 16; b++) {
                        const uint32_t c = (w[i] >> (2 * b)) & 3u;   // 0 -> -x, 1 -> 0 * x, 2 -> +x
#pragma unroll
                        for (int m = 0; m < M; m++) {
                            float xv = xs[xg + m * K + i * 16 + b];
                            // a zero weight still multiplies x, so an infinity or NaN in x gives NaN
                            part[m] += c == 2u ? xv : (c == 0u ? -xv : 0.f * xv);
                        }
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < M; m++)
                acc[m] = fmaf(s, part[m], acc[m]);     // scale once per group
        }
    }
#pragma unroll
    for (int m = 0; m < M; m++) {
        acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], 4);
        acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], 2);
        acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], 1);
    }
    if (j == 0 && n < N) {
#pragma unroll
        for (int m = 0; m < M; m++) {
            if (yt == BQ_F32)
                store_out(static_cast<float *>(y) + m * N + n, acc[m]);
            else if (yt == BQ_BF16)
                store_out(static_cast<__nv_bfloat16 *>(y) + m * N + n, acc[m]);
            else
                store_out(static_cast<__half *>(y) + m * N + n, acc[m]);
        }
    }
}

template <int FMT, int M, typename XT>
cudaError_t launch_simt_t(const GemvArgs &a, cudaStream_t s)
{
    const size_t smem = (size_t)M * (size_t)a.K * sizeof(float);
    const unsigned blocks = (unsigned)((a.N + kRowsPerBlock - 1) / kRowsPerBlock);
    if (smem <= kSimtMaxSmem) {
        auto kern = gemv_simt_kernel<FMT, M, XT, true>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        kern<<<blocks, kSimtThreads, smem, s>>>(static_cast<const XT *>(a.x), a.K, a.words, a.scales, a.N,
                                                a.y, a.yt);
    } else {
        gemv_simt_kernel<FMT, M, XT, false><<<blocks, kSimtThreads, 0, s>>>(
            static_cast<const XT *>(a.x), a.K, a.words, a.scales, a.N, a.y, a.yt);
    }
    return cudaGetLastError();
}

template <int FMT, typename XT>
cudaError_t launch_simt_m(const GemvArgs &a, cudaStream_t s)
{
    switch (a.M) {
    case 1: return launch_simt_t<FMT, 1, XT>(a, s);
    case 2: return launch_simt_t<FMT, 2, XT>(a, s);
    case 3: return launch_simt_t<FMT, 3, XT>(a, s);
    case 4: return launch_simt_t<FMT, 4, XT>(a, s);
    case 5: return launch_simt_t<FMT, 5, XT>(a, s);
    case 6: return launch_simt_t<FMT, 6, XT>(a, s);
    case 7: return launch_simt_t<FMT, 7, XT>(a, s);
    default: return launch_simt_t<FMT, 8, XT>(a, s);
    }
}

}  // namespace

template <int FMT>
cudaError_t launch_simt_x(const GemvArgs &a, cudaStream_t s)
{
    if (a.xt == BQ_F16)
        return launch_simt_m<FMT, __half>(a, s);
    if (a.xt == BQ_BF16)
        return launch_simt_m<FMT, __nv_bfloat16>(a, s);
    return launch_simt_m<FMT, float>(a, s);
}

cudaError_t launch_gemv_simt(const GemvArgs &a, cudaStream_t s)
{
    if (a.fmt == BQ_BINARY_G128)
        return launch_simt_x<BQ_BINARY_G128>(a, s);
    if (a.fmt == BQ_TERNARY_B3_G128)
        return launch_simt_x<BQ_TERNARY_B3_G128>(a, s);
    return launch_simt_x<BQ_TERNARY_G128>(a, s);
}

// Workspace of the tensor-core path (the digit fragments of x); the SIMT kernel needs none.
size_t gemv_workspace_bytes(int M, int fmt, int64_t N, int64_t K)
{
    return gemv_rows_supported(M, fmt, N, K) ? gemv_rows_workspace_bytes(M, fmt, N, K) : 0;
}

// K a multiple of 1024 and the fragments in shared memory: the integer tensor-core kernel
// (gemv_rows.cu); otherwise the SIMT kernel.
cudaError_t launch_gemv(const GemvArgs &a, cudaStream_t s, unsigned *launches)
{
    if (gemv_rows_supported(a.M, a.fmt, a.N, a.K))
        return launch_gemv_rows(a, s, launches);
    *launches = 1;
    return launch_gemv_simt(a, s);
}

}  // namespace bq
