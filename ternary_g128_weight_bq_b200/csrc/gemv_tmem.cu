// gemv_tmem.cu -- decode GEMV for 5 <= M <= 8 token rows on packed binary-g128 and ternary-g128
// weights, on the fifth-generation tensor cores (tcgen05 kind::i8) with the weight operand in
// tensor memory.
//
// y[m][n] = sum_g s[n][g] * sum_{k in g} (2 b[n][k] - 1) x[m][k]: model card
// "prism-ml/Bonsai-27B-mlx-1bit", sections "Weight representation: Binary g128" and "CUDA
// (NVIDIA GPUs)"; the decode workload of section "Cross-platform throughput".
//
// Per CTA, a ring of TMA stages of 128 rows x 128 bytes of packed words (1024 k), and:
//   * 4 expander warps: each thread takes one weight row and turns each group into s8 values:
//     binary sign bits into b * 2^p (two shifts and eight ANDs per word), ternary codes into
//     {-64, 0, +64} (PRMT through a byte table, four codes per instruction). It writes them with
//     tcgen05.st into a 128-lane x 32-column A tile in tensor memory: four groups per buffer,
//     two buffers;
//   * 1 MMA warp: per group, 4 tcgen05.mma kind::i8 (M 128, N 32, K 32), A from tensor memory
//     and the x digits (B) from shared memory, into one of two half-stage accumulator buffers;
//   * 8 readout warps, two per lane quarter, each taking half of the groups: tcgen05.ld of the
//     row's accumulators, then the digit weights, the -64 sum(X) correction, the group scale
//     and the x factor, summed in fp32 per row and token (the pair meets once per block);
//   * 1 TMA producer warp.
// Binary: x enters as four balanced base-64 digits per (token, group) of X = round(x 2^(21-e)),
// each digit multiplied by 2^(7-p) (negated for p = 7) to match the sign byte's position p. Each
// product is then 128 b d, and sum_d 64^d D_d - 64 sum(X) = 64 sum((2b - 1) X). Ternary: three
// balanced base-256 digits and a zero column, products 64 (c - 1) d. A prep kernel
// builds the B tiles, the factors 2^(e-27) and sum(X) once per call. The work is split
// stream-K over (128-row block, 1024-k stage) units, with the same split-block partial sums
// and counters as gemv_tc.cu.
//
// Why only M >= 5. Per-warp clock counters measured one issuing thread taking about 74 cycles
// per tcgen05.mma at N = 8 (M <= 2) and about 41 at N = 32. A 128 x 32 weight tile (4096
// weights) per instruction then caps M = 1 well below the mma.sync kernel of gemv_tc.cu (binary
// LM head 129 us against 73 us; ternary N = 248320: 145 us against 110 us). At M = 8 the
// mma.sync kernel is itself tensor-bound (32 MMA columns per group), and this kernel is faster:
// N = 20480, K = 5120: binary 24.0 us against 26.4 us, ternary 25.1 us against 26.6 us.
#include <cuda.h>

#include "bq_internal.cuh"
#include "sm100_ptx.cuh"

namespace bq {
namespace {

constexpr int kRows = 128;
constexpr int kStageBytes = kRows * 128;
// a stage is 128 bytes of packed words per row: 8 binary groups or 4 ternary groups
template <int FMT> struct TCfg {
    static constexpr int kGroups = FMT == BQ_BINARY_G128 ? 8 : 4;
    static constexpr int kHalves = kGroups / 4;       // 4-group half stages (the A buffer unit)
};
constexpr int kExpWarps = 4, kOutWarps = 8;
constexpr int kThreads = (2 + kExpWarps + kOutWarps) * 32;
constexpr int kMaxABuf = 3;            // sign-operand buffers of 4 groups (128 columns) each
__host__ __device__ constexpr int abufs(int N) { return N == 32 ? 2 : 3; }
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 227 * 1024;
constexpr int kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__host__ __device__ constexpr int bin_p(int rho) { return rho == 2 || rho == 5 ? 5 : (rho == 0 || rho == 3 || rho == 6 ? 6 : 7); }
__host__ __device__ constexpr int bin_bmul(int rho) { return bin_p(rho) == 5 ? 4 : (bin_p(rho) == 6 ? 2 : -1); }

struct Bars {
    uint64_t full[kMaxStages], empty[kMaxStages];
    uint64_t afull[kMaxABuf], afree[kMaxABuf];
    uint64_t dfull[2], dfree[2];
    uint64_t pfull[4], pfree[4];         // the two readout warps of a lane quarter meet per block
    uint64_t frag, drain;
    uint32_t tmem_base;
    int abort;
};

struct Layout {
    int b_off, fx_off, pair_off, stage_off, bar_off, total;
};

template <int N>
__host__ __device__ inline Layout make_layout(int G, int stages)
{
    Layout L;
    L.b_off = 0;                                         // B tiles [G][N][128 B], SW128 images
    L.fx_off = G * N * 128;                              // f [slots][G], sum(X) [slots][G]
    L.pair_off = L.fx_off + 2 * (N / 4) * G * 4;         // [128 rows][slots] f32
    L.stage_off = (L.pair_off + kRows * (N / 4) * 4 + 1023) / 1024 * 1024;
    L.bar_off = L.stage_off + stages * kStageBytes;
    L.total = L.bar_off + 512 + 1024;
    return L;
}

// s8 sign bytes of one word: register rho holds, in byte b, bit 8b + rho as b * 2^p(rho).
__device__ __forceinline__ void expand_mask(uint32_t w, const uint32_t (&mk)[5], uint32_t *a)
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

__device__ __forceinline__ void tmem_ld_cols(uint32_t ta, uint32_t (&r)[8]) { ptx::tmem_ld_32x32b_x8(ta, r); }
__device__ __forceinline__ void tmem_ld_cols(uint32_t ta, uint32_t (&r)[16]) { ptx::tmem_ld_32x32b_x16(ta, r); }
__device__ __forceinline__ void tmem_ld_cols(uint32_t ta, uint32_t (&r)[32]) { ptx::tmem_ld_32x32b_x32(ta, r); }

// 4 s8 registers of one ternary word (16 codes) through a PRMT byte table: code 0 -> -64, 1 -> 0,
// 2 -> +64, 3 (never written by the pack calls) -> 0. Register j, byte b holds code i(j, b):
// j = 0: 2b, 1: 8 + 2b, 2: 2b + 1, 3: 9 + 2b.
__device__ __forceinline__ void expand_ternary4(uint32_t w, uint32_t *a)
{
    const uint32_t table = 0x004000C0u;
    const uint32_t e = w & 0x33333333u, o = (w >> 2) & 0x33333333u;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(a[0]) : "r"(table), "r"(e));
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(a[1]) : "r"(table), "r"(e >> 16));
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(a[2]) : "r"(table), "r"(o));
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(a[3]) : "r"(table), "r"(o >> 16));
}

// Warp-uniform bounded wait (every lane observes the phase).
__device__ __forceinline__ bool wwait(uint64_t *bar, uint32_t parity, volatile int *abort, unsigned int *err)
{
    return __all_sync(0xffffffffu, ptx::mbar_wait_bounded(bar, parity, abort, err, kDevErrTimeout, kWaitLimitNs));
}

// B tiles, factors and sum(X) of (group q, token slot m), one warp. Lane L fills bytes 4 L + b
// (b = 0..3) of the group's 128-byte B rows, i.e. tensor-memory column L of the A tile:
//   binary (expand_mask, L = 8 w + rho): k = 32 w + 8 b + rho; four base-64 digits, each
//     times 2^(7 - p(rho)), and sum(X) for the -64 sum(X) correction;
//   ternary (expand_ternary4, L = 4 w + j): k = 16 w + i(j, b); three base-256 digits and a
//     zero column (the codes enter as {-64, 0, +64}, so no correction).
template <int FMT, int N, typename XT>
__global__ void __launch_bounds__(256)
gemv_tmem_prep_kernel(const XT *__restrict__ x, int M, int64_t K, uint8_t *__restrict__ btile, float *__restrict__ fx,
               unsigned int *__restrict__ counters, int n_counters)
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int kSlots = N / 4;
    const int G = (int)(K / 128);
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < n_counters; i += 256)
            counters[i] = 0u;
    const int item = (int)((blockIdx.x * 256 + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (item >= G * kSlots)
        return;
    const int q = item / kSlots, m = item % kSlots;
    constexpr bool kBin = FMT == BQ_BINARY_G128;
    constexpr int kBits = kBin ? 6 : 8, kDig = kBin ? 4 : 3;
    const int w = kBin ? lane >> 3 : lane >> 2, rho = kBin ? lane & 7 : lane & 3;
    auto kidx = [&](int b) {
        if (kBin)
            return 32 * w + 8 * b + rho;
        const int i = rho == 0 ? 2 * b : rho == 1 ? 8 + 2 * b : rho == 2 ? 2 * b + 1 : 9 + 2 * b;
        return 16 * w + i;
    };
    uint32_t dw[4] = {0u, 0u, 0u, 0u};
    int xs = 0;
    float fac = 0.f;
    if (m < M) {
        float v[4];
#pragma unroll
        for (int b = 0; b < 4; b++)
            v[b] = load_x(x + (int64_t)m * K + 128 * q + kidx(b));
        float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
        for (int o = 16; o; o >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        int e = 0;
        if (amax > 0.f) {
            frexpf(amax, &e);
            e -= 1;
        }
        const int bmul = kBin ? bin_bmul(rho) : 1;
#pragma unroll
        for (int b = 0; b < 4; b++) {
            int X = amax > 0.f ? __float2int_rn(ldexpf(v[b], 21 - e)) : 0;
            xs += kBin ? X : 0;
#pragma unroll
            for (int d = 0; d < kDig; d++) {
                constexpr int kHalf = 1 << (kBits - 1), kMask = (1 << kBits) - 1;
                const int dig = ((X + kHalf) & kMask) - kHalf;
                dw[d] |= ((uint32_t)(dig * bmul) & 0xFFu) << (8 * b);
                X = (X - dig) >> kBits;
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1)
            xs += __shfl_xor_sync(0xffffffffu, xs, o);
        fac = amax > 0.f ? ldexpf(1.f, e - 27) : 0.f;
    }
#pragma unroll
    for (int d = 0; d < 4; d++) {
        const int n = 4 * m + d, j = lane >> 2;
        uint32_t *row = reinterpret_cast<uint32_t *>(btile + ((size_t)q * N + n) * 128);
        row[((j ^ (n & 7)) << 2) + (lane & 3)] = dw[d];
    }
    if (lane == 0) {
        fx[m * G + q] = fac;
        fx[kSlots * G + m * G + q] = (float)xs;
    }
}

template <typename T>
__device__ __forceinline__ void store_y(void *y, int yt, int64_t idx, float v)
{
    if (yt == BQ_F32)
        store_out(static_cast<float *>(y) + idx, v);
    else if (yt == BQ_BF16)
        store_out(static_cast<__nv_bfloat16 *>(y) + idx, v);
    else
        store_out(static_cast<__half *>(y) + idx, v);
}

template <int FMT, int N>
__global__ void __launch_bounds__(kThreads, 1)
gemv_tmem_kernel(const __grid_constant__ CUtensorMap tmap_w, const uint16_t *__restrict__ scales, int M,
               int64_t Nr, int64_t K, void *__restrict__ y, int yt, float *__restrict__ part,
               unsigned int *__restrict__ counters, const uint8_t *__restrict__ btile_g,
               const float *__restrict__ fx_g, int64_t U, int C, int stages, uint32_t one,
               unsigned int *dev_status)
{
    constexpr int kSlots = N / 4;
    constexpr int kGroups = TCfg<FMT>::kGroups, kHalves = TCfg<FMT>::kHalves;
    constexpr bool kBin = FMT == BQ_BINARY_G128;
    const int G = (int)(K / 128);
    const Layout L = make_layout<N>(G, stages);
    const int S = stages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *bs = smem + L.b_off;
    float *fx = reinterpret_cast<float *>(smem + L.fx_off);
    Bars *bars = reinterpret_cast<Bars *>(smem + L.bar_off);
    volatile int *abort = &bars->abort;
    unsigned int *err = dev_status + kSlotErrBits;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t Pn = gridDim.x;
    const int64_t u0 = (int64_t)blockIdx.x * U / Pn, u1 = ((int64_t)blockIdx.x + 1) * U / Pn;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            ptx::mbar_init(&bars->full[s], 1);
            ptx::mbar_init(&bars->empty[s], kExpWarps);
        }
        for (int i = 0; i < kMaxABuf; i++) {
            ptx::mbar_init(&bars->afull[i], kExpWarps);
            ptx::mbar_init(&bars->afree[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            ptx::mbar_init(&bars->dfull[i], 1);
            ptx::mbar_init(&bars->dfree[i], kOutWarps);
        }
        for (int i = 0; i < 4; i++) {
            ptx::mbar_init(&bars->pfull[i], 1);
            ptx::mbar_init(&bars->pfree[i], 1);
        }
        ptx::mbar_init(&bars->frag, 1);
        ptx::mbar_init(&bars->drain, 1);
        bars->abort = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(&bars->tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    // tensor memory: NA sign-operand buffers of 4 groups x 32 columns, then 2 accumulator
    // buffers of 4 groups x N columns (a half stage each)
    constexpr int NA = abufs(N);
    const uint32_t a_base = tmem, d_base = tmem + 128 * NA;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == 0) {
        // ------------------------------------------------------------- TMA producer
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tmap_w);
            int64_t it = 0;
            int s = 0;
            uint32_t ph = 0;
            int64_t rb = u0 / C;
            int c = (int)(u0 % C);
            for (int64_t u = u0; u < u1; u++, it++) {
                if (!ptx::mbar_wait_bounded_sleep(&bars->empty[s], ph ^ 1, abort, err, kDevErrTimeout, kWaitLimitNs))
                    break;
                ptx::mbar_arrive_expect_tx(&bars->full[s], kStageBytes);
                ptx::tma_load_2d(smem + L.stage_off + s * kStageBytes, &tmap_w, &bars->full[s], c * 32,
                                 (int32_t)(rb * kRows));
                if (++s == S) {
                    s = 0;
                    ph ^= 1;
                }
                if (++c == C) {
                    c = 0;
                    rb++;
                }
            }
            for (int64_t k = it > S ? it - S : 0; k < it; k++) {
                volatile int no_abort = 0;
                ptx::mbar_wait_bounded(&bars->full[k % S], (uint32_t)((k / S) & 1), &no_abort, err,
                                       kDevErrTimeout, kWaitLimitNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            // the B tiles and factors are written by the prep kernel launched just before this one
            asm volatile("griddepcontrol.wait;" ::: "memory");
            int ra0 = 0, ra1 = C, rb1 = 0;
            if (u1 - u0 < C) {
                const int cA = (int)(u0 % C), cB = (int)((u1 - 1) % C);
                ra0 = cA;
                if (cA <= cB) {
                    ra1 = cB + 1;
                } else {
                    ra1 = C;
                    rb1 = cB + 1;
                }
            }
            constexpr uint32_t kChunkB = kGroups * N * 128;
            const uint32_t fx_bytes = (uint32_t)(2 * kSlots * G * 4);
            ptx::mbar_arrive_expect_tx(&bars->frag, (uint32_t)(ra1 - ra0 + rb1) * kChunkB + fx_bytes);
            ptx::bulk_load(bs + (size_t)ra0 * kChunkB, btile_g + (size_t)ra0 * kChunkB, (uint32_t)(ra1 - ra0) * kChunkB,
                           &bars->frag);
            if (rb1 > 0)
                ptx::bulk_load(bs, btile_g, (uint32_t)rb1 * kChunkB, &bars->frag);
            ptx::bulk_load(fx, fx_g, fx_bytes, &bars->frag);
            constexpr uint32_t idesc = ptx::umma_idesc_s8(kRows, N);
            bool ok = ptx::mbar_wait_bounded(&bars->frag, 0, abort, err, kDevErrTimeout, kWaitLimitNs);
            int64_t hs = 0;
            for (int64_t u = u0; ok && u < u1; u++) {
                const int c = (int)(u % C);
                for (int h = 0; ok && h < kHalves; h++, hs++) {
                    const int ab = (int)(hs % NA), db = (int)(hs & 1);
                    ok = ptx::mbar_wait_bounded(&bars->afull[ab], (uint32_t)((hs / NA) & 1), abort, err,
                                                kDevErrTimeout, kWaitLimitNs) &&
                         ptx::mbar_wait_bounded(&bars->dfree[db], (uint32_t)(((hs >> 1) & 1) ^ 1), abort, err,
                                                kDevErrTimeout, kWaitLimitNs);
                    if (!ok)
                        break;
                    ptx::tc_fence_after();
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const int q = kGroups * c + 4 * h + i;
                        const uint64_t bd = ptx::sw128_kmajor_desc(ptx::smem_u32(bs + (size_t)q * N * 128));
#pragma unroll
                        for (int j = 0; j < 4; j++)      // K step j: 32 k = 32 bytes further along the B rows
                            ptx::umma_i8_ts(d_base + 4 * N * db + N * i, a_base + 128 * ab + 32 * i + 8 * j, bd + 2 * j,
                                            idesc, j);
                    }
                    ptx::umma_commit(&bars->afree[ab]);
                    ptx::umma_commit(&bars->dfull[db]);
                }
            }
            // every issued MMA must be done before tensor memory is released
            ptx::umma_commit(&bars->drain);
            volatile int no_abort = 0;
            ptx::mbar_wait_bounded(&bars->drain, 0, &no_abort, err, kDevErrTimeout, kWaitLimitNs);
            // the fragment copy must have landed before the CTA exits
            ptx::mbar_wait_bounded(&bars->frag, 0, &no_abort, err, kDevErrTimeout, kWaitLimitNs);
        }
    } else if (warp < 2 + kExpWarps) {
        // ------------------------------------------------------------- expanders
        const int qd = warp & 3;
        const int r = 32 * qd + lane;
        const uint32_t mk[5] = {one * 8u, one * 64u, one * 0x20202020u, one * 0x40404040u, one * 0x80808080u};
        int s = 0;
        uint32_t ph = 0;
        int64_t hs = 0;
        bool ok = true;
        for (int64_t u = u0; ok && u < u1; u++) {
            ok = wwait(&bars->full[s], ph, abort, err);
            if (!ok)
                break;
            const uint8_t *stage = smem + L.stage_off + s * kStageBytes + r * 128;
            for (int h = 0; h < kHalves; h++, hs++) {
                const int ab = (int)(hs % NA);
                ok = wwait(&bars->afree[ab], (uint32_t)(((hs / NA) & 1) ^ 1), abort, err);
                if (!ok)
                    break;
                ptx::tc_fence_after();
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int qs = 4 * h + i;
                    uint32_t a[32];
                    if (kBin) {                                  // 4 words: 16-byte chunk qs
                        const uint4 wv = *reinterpret_cast<const uint4 *>(stage + ((qs ^ (r & 7)) << 4));
                        expand_mask(wv.x, mk, a);
                        expand_mask(wv.y, mk, a + 8);
                        expand_mask(wv.z, mk, a + 16);
                        expand_mask(wv.w, mk, a + 24);
                    } else {                                     // 8 words: chunks 2 qs, 2 qs + 1
                        const uint4 w0 = *reinterpret_cast<const uint4 *>(stage + (((2 * qs) ^ (r & 7)) << 4));
                        const uint4 w1 = *reinterpret_cast<const uint4 *>(stage + (((2 * qs + 1) ^ (r & 7)) << 4));
                        expand_ternary4(w0.x, a);
                        expand_ternary4(w0.y, a + 4);
                        expand_ternary4(w0.z, a + 8);
                        expand_ternary4(w0.w, a + 12);
                        expand_ternary4(w1.x, a + 16);
                        expand_ternary4(w1.y, a + 20);
                        expand_ternary4(w1.z, a + 24);
                        expand_ternary4(w1.w, a + 28);
                    }
                    ptx::tmem_st_32x32b_x32(a_base + ((uint32_t)(32 * qd) << 16) + 128 * ab + 32 * i, a);
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    ptx::mbar_arrive(&bars->afull[ab]);
            }
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(&bars->empty[s]);
            if (++s == S) {
                s = 0;
                ph ^= 1;
            }
        }
    } else {
        // ------------------------------------------------------------- readout
        const int qd = warp & 3, ro = (warp - 2 - kExpWarps) >> 2;   // two readout warps per lane quarter
        const int r = 32 * qd + lane;
        bool ok = wwait(&bars->frag, 0, abort, err);
        float *pair = reinterpret_cast<float *>(smem + L.pair_off) + (size_t)r * kSlots;
        const float *fq = fx;                            // f [slot][G]
        const float *xq = fx + kSlots * G;               // sum(X) [slot][G]
        int64_t hs = 0;
        int bi = 0;                                      // block index within this CTA
        for (int64_t rb = u0 / C; ok && rb * C < u1; rb++, bi++) {
            const int c_lo = (int)(rb == u0 / C ? u0 % C : 0);
            const int c_hi = (int)((rb + 1) * C <= u1 ? C : u1 - rb * C);
            const int64_t n = rb * kRows + r;
            const bool nok = n < Nr;
            float acc[kSlots];
#pragma unroll
            for (int m = 0; m < kSlots; m++)
                acc[m] = 0.f;
            for (int c = c_lo; ok && c < c_hi; c++) {
                uint32_t sw[4] = {0u, 0u, 0u, 0u};
                if (nok && kBin) {
                    const uint4 sv = __ldg(reinterpret_cast<const uint4 *>(scales + n * G + kGroups * c));
                    sw[0] = sv.x; sw[1] = sv.y; sw[2] = sv.z; sw[3] = sv.w;
                } else if (nok) {
                    const uint2 sv = __ldg(reinterpret_cast<const uint2 *>(scales + n * G + kGroups * c));
                    sw[0] = sv.x; sw[1] = sv.y;
                }
#pragma unroll
                for (int h = 0; h < kHalves; h++, hs++) {
                    const int db = (int)(hs & 1);
                    ok = wwait(&bars->dfull[db], (uint32_t)((hs >> 1) & 1), abort, err);
                    if (!ok)
                        break;
                    ptx::tc_fence_after();
                    // 32 accumulator columns (32 / N groups) per tensor-memory load; readout warp ro
                    // of the quarter takes loads ro, ro + 2, ... of the half stage
#pragma unroll
                    for (int g0 = (32 / N) * ro; g0 < 4; g0 += 2 * (32 / N)) {
                        uint32_t dv[32];
                        ptx::tmem_ld_32x32b_x32(d_base + ((uint32_t)(32 * qd) << 16) + 4 * N * db + N * g0, dv);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int gl = 0; gl < 32 / N; gl++) {
                            const int i = 4 * h + g0 + gl;       // group within the stage
                            const __half2 hp = *reinterpret_cast<const __half2 *>(&sw[i >> 1]);
                            const float sg = (i & 1) ? __high2float(hp) : __low2float(hp);
                            const int q = kGroups * c + i;
#pragma unroll
                            for (int m = 0; m < kSlots; m++) {
                                const uint32_t *dm = dv + N * gl + 4 * m;
                                constexpr float kW = kBin ? 64.f : 256.f;    // digit weight
                                float v = (float)(int)dm[3];
                                v = fmaf(v, kW, (float)(int)dm[2]);
                                v = fmaf(v, kW, (float)(int)dm[1]);
                                v = fmaf(v, kW, (float)(int)dm[0]);
                                if (kBin)
                                    v = fmaf(-64.f, xq[m * G + q], v);
                                acc[m] = fmaf(sg * fq[m * G + q], v, acc[m]);
                            }
                        }
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        ptx::mbar_arrive(&bars->dfree[db]);
                }
            }
            if (!ok)
                break;
            // the second readout warp of the quarter hands its sums to the first
            if (ro == 1) {
                if (bi > 0 && !wwait(&bars->pfree[qd], (uint32_t)((bi - 1) & 1), abort, err))
                    break;
#pragma unroll
                for (int m = 0; m < kSlots; m++)
                    pair[m] = acc[m];
                __syncwarp();
                if (lane == 0)
                    ptx::mbar_arrive(&bars->pfull[qd]);
                continue;
            }
            if (!wwait(&bars->pfull[qd], (uint32_t)(bi & 1), abort, err))
                break;
#pragma unroll
            for (int m = 0; m < kSlots; m++)
                acc[m] += pair[m];
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(&bars->pfree[qd]);
            const bool whole = c_lo == 0 && c_hi == C;
            const int64_t x0 = rb * C, x1 = rb * C + C;
            const int64_t i_first = (x0 + 1) * Pn / U + (((x0 + 1) * Pn) % U != 0) - 1;
            const int64_t i_last = x1 * Pn / U + ((x1 * Pn) % U != 0) - 1;
            const int nseg = (int)(i_last - i_first + 1);
            const int end = rb == u0 / C ? 0 : 1;
            if (whole) {
#pragma unroll
                for (int m = 0; m < kSlots; m++)
                    if (nok && m < M)
                        store_y<float>(y, yt, (int64_t)m * Nr + n, acc[m]);
            } else {
#pragma unroll
                for (int m = 0; m < kSlots; m++)
                    if (m < M)
                        part[(((int64_t)blockIdx.x * 2 + end) * kRows + r) * M + m] = acc[m];
                __syncwarp();
                int last = 0;
                if (lane == 0)
                    last = ptx::atom_add_acq_rel_gpu(counters + i_first * 4 + qd, 1u) == (unsigned)(nseg - 1);
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last) {
                    __syncwarp();
                    float v[kSlots];
#pragma unroll
                    for (int m = 0; m < kSlots; m++)
                        v[m] = 0.f;
                    for (int sg0 = 0; sg0 < nseg; sg0 += 8) {
                        float pv[8][kSlots];
#pragma unroll
                        for (int j = 0; j < 8; j++) {
                            const int sgi = sg0 + j;
                            const int64_t i = i_first + sgi;
                            const int slot_i = sgi == 0 && i * U / Pn != x0 ? 1 : 0;
                            const float *pp = part + ((i * 2 + slot_i) * kRows + r) * M;
#pragma unroll
                            for (int m = 0; m < kSlots; m++)
                                pv[j][m] = sgi < nseg && m < M ? __ldcg(pp + m) : 0.f;
                        }
#pragma unroll
                        for (int j = 0; j < 8; j++)
#pragma unroll
                            for (int m = 0; m < kSlots; m++)
                                v[m] += pv[j][m];
                    }
#pragma unroll
                    for (int m = 0; m < kSlots; m++)
                        if (nok && m < M)
                            store_y<float>(y, yt, (int64_t)m * Nr + n, v[m]);
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_tmem()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

int sm_count_tmem()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

// accumulator columns: 4 per token slot (four binary digits, or three ternary ones and a zero);
// this kernel runs for M >= 5 only, so always 8 slots
int n_cols(int fmt, int M)
{
    (void)fmt;
    (void)M;
    return 32;
}

template <int N>
int plan_stages_tmem(int G)
{
    for (int s = kMaxStages; s >= 2; s--)
        if (make_layout<N>(G, s).total <= kSmemLimit)
            return s;
    return 0;
}

int stages_tmem(int fmt, int M, int G)
{
    (void)fmt;
    (void)M;
    return plan_stages_tmem<32>(G);
}

struct PlanTmem {
    int N, stages, grid;
    int64_t NB, C, U;
    size_t part_bytes, counter_bytes, b_bytes, fx_bytes;
    int n_counters;
};

PlanTmem make_plan_tmem(int M, int fmt, int64_t Nr, int64_t K)
{
    PlanTmem p;
    p.N = n_cols(fmt, M);
    const int G = (int)(K / 128);
    p.stages = stages_tmem(fmt, M, G);
    p.NB = (Nr + kRows - 1) / kRows;
    p.C = K / (fmt == BQ_BINARY_G128 ? 1024 : 512);   // stages of 128 bytes per row
    p.U = p.NB * p.C;
    const int64_t sms = sm_count_tmem();
    p.grid = (int)(p.U < sms ? p.U : sms);
    auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
    p.part_bytes = al((size_t)p.grid * 2 * kRows * M * 4);
    p.n_counters = p.grid * 4;
    p.counter_bytes = al((size_t)p.n_counters * 4);
    p.b_bytes = al((size_t)G * p.N * 128);
    p.fx_bytes = al((size_t)2 * (p.N / 4) * G * 4);
    return p;
}

template <int FMT, int N, typename XT>
cudaError_t launch_tmem_t(const GemvArgs &a, const PlanTmem &pl, cudaStream_t s)
{
    EncodeTiledFn enc = encode_fn_tmem();
    if (!enc)
        return cudaErrorNotSupported;
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    float *part = reinterpret_cast<float *>(ws);
    unsigned int *counters = reinterpret_cast<unsigned int *>(ws + pl.part_bytes);
    uint8_t *btile = ws + pl.part_bytes + pl.counter_bytes;
    float *fx = reinterpret_cast<float *>(ws + pl.part_bytes + pl.counter_bytes + pl.b_bytes);
    CUtensorMap mw;
    const cuuint64_t wpr = (cuuint64_t)(FMT == BQ_BINARY_G128 ? a.K / 32 : a.K / 16);
    cuuint64_t wdims[2] = {wpr, (cuuint64_t)a.N};
    cuuint64_t wstr[1] = {wpr * 4};
    cuuint32_t wbox[2] = {32, (cuuint32_t)kRows};        // 128 bytes x 128 rows
    cuuint32_t est[2] = {1, 1};
    CUresult r = enc(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(a.words), wdims, wstr, wbox, est,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const int G = (int)(a.K / 128);
    const int smem = make_layout<N>(G, pl.stages).total;
    auto kern = gemv_tmem_kernel<FMT, N>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t pcfg = {};
    const int items = G * (N / 4);
    pcfg.gridDim = dim3((unsigned)((items * 32 + 255) / 256));
    pcfg.blockDim = dim3(256);
    pcfg.stream = s;
    pcfg.attrs = attr;
    pcfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&pcfg, gemv_tmem_prep_kernel<FMT, N, XT>, static_cast<const XT *>(a.x), a.M, a.K, btile, fx,
                           counters, pl.n_counters);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mw, reinterpret_cast<const uint16_t *>(a.scales), a.M, a.N, a.K, a.y, a.yt,
                              part, counters, (const uint8_t *)btile, (const float *)fx, pl.U, (int)pl.C, pl.stages,
                              1u, a.dev_status);
}

template <int FMT, typename XT>
cudaError_t launch_tmem_n(const GemvArgs &a, const PlanTmem &pl, cudaStream_t s)
{
    return launch_tmem_t<FMT, 32, XT>(a, pl, s);
}

}  // namespace

// 5 <= M <= 8 (binary or ternary), K a multiple of 1024 and the B tiles of all of K in shared
// memory next to at least two stages. Below M = 5 the mma.sync kernel of gemv_tc.cu is faster:
// ternary N = 20480, K = 5120: 18.1 us against 19.6 (M = 1), 21.3 against 22.3 (M = 4), while
// M = 8 is 25.1 here against 26.6 there.
bool gemv_tmem_supported(int M, int fmt, int64_t K)
{
    if (M < 5 || M > 8 || K % 1024 != 0)
        return false;
    if (fmt != BQ_BINARY_G128 && fmt != BQ_TERNARY_G128)
        return false;
    return stages_tmem(fmt, M, (int)(K / 128)) >= 2;
}

size_t gemv_tmem_workspace_bytes(int M, int fmt, int64_t N, int64_t K)
{
    PlanTmem p = make_plan_tmem(M, fmt, N, K);
    return p.part_bytes + p.counter_bytes + p.b_bytes + p.fx_bytes;
}

cudaError_t launch_gemv_tmem(const GemvArgs &a, cudaStream_t s)
{
    PlanTmem pl = make_plan_tmem(a.M, a.fmt, a.N, a.K);
    if (a.fmt == BQ_BINARY_G128)
        return a.xt == BQ_F16 ? launch_tmem_n<BQ_BINARY_G128, __half>(a, pl, s)
                              : launch_tmem_n<BQ_BINARY_G128, __nv_bfloat16>(a, pl, s);
    return a.xt == BQ_F16 ? launch_tmem_n<BQ_TERNARY_G128, __half>(a, pl, s)
                          : launch_tmem_n<BQ_TERNARY_G128, __nv_bfloat16>(a, pl, s);
}

}  // namespace bq
