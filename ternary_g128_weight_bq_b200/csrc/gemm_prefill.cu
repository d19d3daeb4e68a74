// gemm_prefill.cu -- prefill GEMM Y[M][N] = X[M][K] * W^T on packed binary-g128 /
// ternary-g128 weights, on the fifth-generation tensor cores (tcgen05, fp32 accumulation in
// tensor memory).
//
// Model card "prism-ml/Bonsai-27B-mlx-1bit", section "CUDA (NVIDIA GPUs)": the kernel unpacks
// the sign codes inside the matrix product and applies the group scale; the model is never
// expanded to a dense FP16 tensor in memory. Section "Cross-platform throughput": pp512 (a
// 512-token prompt) is the compute-bound phase. Ternary: "Ternary Bonsai 27B vs ..." article
// (wmrh.cn), PP512 row of its throughput table.
//
// One CTA computes a 128 (weight rows) x BN (tokens) tile of Y^T:
//   * warp 0, one lane: TMA loads of the X tile [BN tokens x 64 k] per k-block into a ring
//     of shared-memory stages (128-byte swizzle, zero fill past M); warp 0 also owns TMEM.
//   * warps 2-9 (256 threads, two per weight row, each taking half of a k-block): read the
//     row's packed bits and its group scale straight from global memory, expand every pair of
//     weights to +-s (binary) or {-s, 0, +s} (ternary, from 2-bit codes or base-3 bytes) in the
//     operand type with a few integer or packed 16-bit float operations (expand_pairs,
//     expand_pairs_b3), and write the 128 x 64 A tile with
//     tcgen05.st straight into tensor memory (a ring of A stages next to the accumulator), so
//     A needs no shared memory and no proxy fence. The scale is folded into the operand, so a
//     group needs no separate rescaling. The operand type is always fp16, where +-s is exact
//     (an fp16 scale has 11 significant bits; bf16 would keep 8, a relative error of up to
//     2^-8 per weight, about twice the 2e-3 sum|x s| tolerance when every term errs the same
//     way). Per-CTA cycle counters showed the MMA issuer waiting on this
//     step for more than half of its loop while it wrote shared memory; with a 256-entry
//     sign-mask table in shared memory the table's bank-conflicted lookups still held the
//     load/store pipe at about 64% busy, next to the X tiles that the tensor cores read there.
//   * warp 1, one lane: issues 4 tcgen05.mma (128 x BN x 16, A from tensor memory, X from
//     shared memory) per k-block into the TMEM accumulator and commits each stage back to the
//     producers.
//   * warps 2-9 then read the accumulator with tcgen05.ld (lane = weight row, column =
//     token; the two warps of a lane quarter take alternate 32-token blocks), convert to the
//     output type into a [BN tokens][128 rows] tile in the (now idle) X ring, and one thread
//     writes the tile with a TMA tensor store that clips at M and N. When a row of Y is not a
//     whole number of 16-byte units, each warp stores its 32-row segments directly instead.
// bf16 x: a conversion pass (prefill_x16_kernel) first writes x * 2^e_m as fp16 into the
// workspace, e_m a power of two per token row that puts the row's largest finite magnitude in
// [2^14, 2^15). A bf16 value has 8 significant bits, so every element within 2^31 of its row's
// largest magnitude is exact in fp16; smaller ones round to fp16's subnormal spacing (error at
// most 2^-39 of the row's largest magnitude). The epilogue (and the split-tail reduce)
// multiplies each token's fp32 result by 2^-e_m, which is exact.
// Tiles fill whole waves of one tile per CTA; a short last wave is split along K over the idle
// SMs (fp32 partials in the workspace, added in split order by prefill_reduce_kernel). The
// split grid and the reduce are programmatic dependent launches: the split CTAs take SMs as
// the whole-tile grid frees them, and each dependent grid completes only after its
// predecessor, so the stream order seen by later work is unchanged.
// The expanded weights exist only on chip. Every mbarrier wait is bounded: after 2 s (or the
// shorter test limit of bq_debug_set_wait_limit_ns, for the pipeline waits) the kernel records
// kDevErrTimeout, lets its copies and MMAs drain (those waits keep 2 s), frees TMEM and returns.
#include <cuda.h>

#include <cstring>

#include "b3.cuh"
#include "bq_internal.cuh"
#include "sm100_ptx.cuh"

namespace bq {
namespace {

constexpr int kBM = 128;              // weight rows per tile (MMA M)
constexpr int kBK = 64;               // k per stage: one 128-byte swizzle row of 16-bit values
constexpr int kDequantWarps = 8;      // kParts per weight row: each expands 1/kParts of a k-block
                                      // (16 warps, four per row, measured slower)
constexpr int kParts = kDequantWarps / 4;
constexpr int kThreads = (2 + kDequantWarps) * 32;
constexpr uint64_t kWaitLimitNs = kWaitLimitDefaultNs;   // drain waits before exit

// X tiles come by TMA into a shared-memory ring; A tiles (the +-s operand) are written by the
// dequant warps straight into tensor memory, next to the accumulator: D in columns [0, BN),
// A stage a in columns BN + 32 a (64 k of 16-bit values = 32 columns per lane).
template <int BN> struct Cfg {
    static constexpr int kXStages = BN == 256 ? 6 : 8;
    static constexpr int kAStages = BN == 256 ? 6 : 8;
    static constexpr int kXBytes = BN * 128;          // X stage: BN rows x 128 B
    static constexpr int kBarOffset = kXStages * kXBytes;
    // barriers + alignment slack; at least 116 KB so that one CTA holds the SM (and all 512
    // tensor-memory columns)
    static constexpr int kSmemUsed = kBarOffset + 512 + 1024;
    static constexpr int kSmem = kSmemUsed > 116 * 1024 ? kSmemUsed : 116 * 1024;
    static constexpr uint32_t kTmemCols = 512;
    // the epilogue stages a [BN][128] output tile (at most fp32) in the X ring
    static_assert(BN * kBM * 4 <= kXStages * kXBytes, "output staging tile exceeds the X ring");
};

struct Bars {
    uint64_t full_x[8];
    uint64_t empty_x[8];
    uint64_t full_a[8];
    uint64_t empty_a[8];
    uint64_t acc_full;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int staged;   // epilogue warps whose slice of the output tile is in shared memory
};

// Warp-uniform bounded wait: lane 0 waits, the verdict is broadcast, then every lane
// observes the (already completed) phase itself so that it acquires the producer's writes.
// All lanes return the same value, so later warp-collective instructions stay converged.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort, unsigned int *err,
                                          uint64_t limit)
{
    bool ok = true;
    if ((threadIdx.x & 31) == 0)
        ok = ptx::mbar_wait_bounded(bar, parity, abort, err, kDevErrTimeout, limit);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok)
        ok = ptx::mbar_wait_bounded(bar, parity, abort, err, kDevErrTimeout, limit);
    return __all_sync(0xffffffffu, ok);
}

// Column c of a thread's A slice holds weights 2c (low half) and 2c+1 (high half) as +-s or
// {-s, 0, +s} in fp16; s2 is s in both halves. Plain ALU work, no table: the shared-memory
// pipe stays with the X tiles that the tensor cores read.
//   binary: the two sign bits of a pair are moved to bits 15 and 31 (a set bit means -s) and
//     XORed into s2; for a 16-bit slice the odd bits are first lifted by 15, so that one shift
//     per pair puts both in place.
//   ternary: the two codes of a pair go to the low bits of the two halves of the fp16 value
//     1024, where one unit of the last place is 1; then (1024 + c) - 1025 = c - 1 and
//     (c - 1) * s are both exact. A code 3 (never written by the pack calls) gives +2s.
template <int FMT, int COLS>
__device__ __forceinline__ void expand_pairs(uint2 wv, uint32_t s2, uint32_t (&av)[COLS])
{
    if (FMT == BQ_BINARY_G128) {
        const uint32_t nw = ~wv.x;
#pragma unroll
        for (int hh = 0; hh < COLS / 8; hh++) {
            const uint32_t x = nw >> (16 * hh);
            const uint32_t d = (x & 0x5555u) | ((x & 0xAAAAu) << 15);
#pragma unroll
            for (int j = 0; j < 8; j++)
                av[8 * hh + j] = s2 ^ ((d << (15 - 2 * j)) & 0x80008000u);
        }
    } else {
        constexpr uint32_t kMagic = 0x64006400u;                           // 1024 | 1024
        constexpr uint32_t kMagic1 = 0x64016401u;                          // 1025 | 1025
#pragma unroll
        for (int wi = 0; wi < COLS / 8; wi++) {
            const uint32_t w = wi ? wv.y : wv.x;
            const uint32_t e = w & 0x33333333u, o = (w >> 2) & 0x33333333u;   // even / odd weights
            const uint32_t p[2] = {__byte_perm(e, o, 0x5410), __byte_perm(e, o, 0x7632)};
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const uint32_t h = ((p[j >> 2] >> (4 * (j & 3))) & 0x00030003u) | kMagic;
                __half2 v = __hsub2(*reinterpret_cast<const __half2 *>(&h),
                                    *reinterpret_cast<const __half2 *>(&kMagic1));
                v = __hmul2(v, *reinterpret_cast<const __half2 *>(&s2));
                av[8 * wi + j] = *reinterpret_cast<const uint32_t *>(&v);
            }
        }
    }
}

// Base-3 storage (b3.cuh). A thread's 32 weights of a k-block are positions 32 V .. 32 V + 31 of
// a group (V = 2 (k-block % 2) + its half of the k-block); they sit in the 8 group bytes
// b3_pf_start(V) .. + 7 (for V = 3: five-code bytes 18..23 and the two four-code bytes), which
// it loads as four 16-bit values (every such offset is even). Code p of a byte q is
// floor(3 ((q 3^p) mod 256) / 256), so the two codes of a pair come from one multiply into
// 16-bit lanes (two when the pair straddles two bytes), a mask, a multiply by 3 and a PRMT that
// puts each code under the exponent bits of the fp16 value 1024; then (1024 + c) - 1025 and the
// product with s are exact, as for the 2-bit codes.
__host__ __device__ constexpr int b3_pf_start(int V) { return V == 0 ? 0 : V == 1 ? 6 : V == 2 ? 12 : 18; }

__device__ __forceinline__ uint32_t prmt_pf(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

template <int V>
__device__ __forceinline__ uint32_t b3_pf_byte(uint2 B, int j)
{
    const int i = j - b3_pf_start(V);                   // 0 .. 7
    return prmt_pf(i < 4 ? B.x : B.y, 0u, 0x4440u + (uint32_t)(i & 3));
}

template <int V>
__device__ __forceinline__ void expand_pairs_b3(uint2 B, uint32_t s2, uint32_t (&av)[16])
{
    constexpr uint32_t kMagic1 = 0x64016401u;           // 1025 | 1025
#pragma unroll
    for (int c = 0; c < 16; c++) {
        const int P = 32 * V + 2 * c;                   // the pair's even position in the group
        const int ja = b3::byte_of(P), jb = b3::byte_of(P + 1);
        const int pa = P - b3::first(ja), pb = P + 1 - b3::first(jb);
        const uint32_t qa = b3_pf_byte<V>(B, ja);
        uint32_t pl;                                    // lanes: q 3^p of the two positions
        if (ja == jb)
            pl = qa * (b3::pow3(pa) + 65536u * b3::pow3(pb));
        else
            pl = b3_pf_byte<V>(B, jb) * (b3::pow3(pb) << 16) + qa * b3::pow3(pa);
        const uint32_t r = (pl & 0x00FF00FFu) * 3u;     // code in bits 8..9 of each lane
        const uint32_t h = prmt_pf(r, 0x64646464u, 0x4341u);   // lanes 1024 + code in fp16
        __half2 v = __hsub2(*reinterpret_cast<const __half2 *>(&h), *reinterpret_cast<const __half2 *>(&kMagic1));
        v = __hmul2(v, *reinterpret_cast<const __half2 *>(&s2));
        av[c] = *reinterpret_cast<const uint32_t *>(&v);
    }
}

__device__ __forceinline__ uint32_t scale_pair(uint16_t s_f16) { return (uint32_t)s_f16 | ((uint32_t)s_f16 << 16); }

// floor(log2 a) of a finite a > 0, from its bits (subnormals included).
__device__ __forceinline__ int ilog2_pos(float a)
{
    const uint32_t u = __float_as_uint(a);
    return u >= 0x00800000u ? (int)(u >> 23) - 127 : -118 - (int)__clz(u);
}

// 2^k as a float for k in [-149, 127] (exact; subnormal below -126), 0 below.
__device__ __forceinline__ float pow2_float(int k)
{
    if (k >= -126)
        return __uint_as_float((uint32_t)(k + 127) << 23);
    return k >= -149 ? __uint_as_float(1u << (k + 149)) : 0.f;
}

// bf16 x -> fp16 x * 2^e_m, one block per token row m: e_m puts the row's largest finite
// magnitude in [2^14, 2^15) (e_m = 0 for a row with no finite non-zero value), and tok_fac[m]
// = 2^-e_m undoes it on the fp32 results. Non-finite values stay non-finite. K is a multiple
// of 128, so every thread moves whole 16-byte chunks of 8 values.
constexpr int kX16Threads = 256;

__global__ void __launch_bounds__(kX16Threads)
prefill_x16_kernel(const __nv_bfloat16 *__restrict__ x, int64_t K, __half *__restrict__ x16,
                   float *__restrict__ tok_fac)
{
    // the GEMM grid may set itself up meanwhile; it waits for this grid before reading x16
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ float wmax[kX16Threads / 32];
    const int64_t m = blockIdx.x;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + m * K);
    uint4 *dst = reinterpret_cast<uint4 *>(x16 + m * K);
    const int chunks = (int)(K / 8);
    // rows up to kHeld chunks per thread (K <= 8192) are read once and kept in registers
    constexpr int kHeld = 4;
    uint4 held[kHeld];
    float amax = 0.f;
    auto absmax = [&](const uint4 &v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
            if (isfinite(f.x))
                amax = fmaxf(amax, fabsf(f.x));
            if (isfinite(f.y))
                amax = fmaxf(amax, fabsf(f.y));
        }
    };
#pragma unroll
    for (int j = 0; j < kHeld; j++) {
        const int c = threadIdx.x + j * kX16Threads;
        held[j] = c < chunks ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < kHeld; j++)
        absmax(held[j]);
    for (int c = threadIdx.x + kHeld * kX16Threads; c < chunks; c += kX16Threads)
        absmax(__ldg(src + c));
#pragma unroll
    for (int o = 16; o; o >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0)
        wmax[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = wmax[0];
#pragma unroll
    for (int i = 1; i < kX16Threads / 32; i++)
        amax = fmaxf(amax, wmax[i]);
    // e = 14 - floor(log2 amax) puts amax 2^e in [2^14, 2^15); the factor 2^e is applied as two
    // exact power-of-two multiplies (e reaches 147 for the smallest bf16 subnormal)
    const int e = amax > 0.f ? 14 - ilog2_pos(amax) : 0;
    const float f1 = pow2_float(e < 127 ? e : 127), f2 = pow2_float(e > 127 ? e - 127 : 0);
    auto convert = [&](const uint4 &v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
            const __half2 h = __floats2half2_rn(f.x * f1 * f2, f.y * f1 * f2);
            o[i] = *reinterpret_cast<const uint32_t *>(&h);
        }
        return make_uint4(o[0], o[1], o[2], o[3]);
    };
#pragma unroll
    for (int j = 0; j < kHeld; j++) {
        const int c = threadIdx.x + j * kX16Threads;
        if (c < chunks)
            dst[c] = convert(held[j]);
    }
    for (int c = threadIdx.x + kHeld * kX16Threads; c < chunks; c += kX16Threads)
        dst[c] = convert(__ldg(src + c));
    if (threadIdx.x == 0)
        tok_fac[m] = pow2_float(-e);       // exact: -e is in [-147, 113]
}

// tok_fac: the per-token factor 2^-e_m of bf16 x (NULL for fp16 x, which is used as it is).
template <int FMT, int BN>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_y, int y_tma,
               const uint32_t *__restrict__ words,
               const uint16_t *__restrict__ scales, int64_t M, int64_t N, int64_t K, void *__restrict__ y,
               int yt, int tiles_m, int tile0, int splits, float *__restrict__ part,
               const float *__restrict__ tok_fac, unsigned int *dev_status, uint64_t wait_ns)
{
    using C = Cfg<BN>;
    constexpr int SX = C::kXStages, SA = C::kAStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *xs = smem;                                         // SX x kXBytes
    Bars *bars = reinterpret_cast<Bars *>(smem + C::kBarOffset);
    volatile int *abort = &bars->abort;
    unsigned int *err = dev_status + kSlotErrBits;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // CTA b takes tile tile0 + b / splits (token tile = tile % tiles_m, row block = tile /
    // tiles_m) and k-blocks [kb0, kb1) of it: all of K unless the tile is split
    const int tile = tile0 + (int)blockIdx.x / splits, split = (int)blockIdx.x % splits;
    const int64_t m0 = (int64_t)(tile % tiles_m) * BN;
    const int64_t n0 = (int64_t)(tile / tiles_m) * kBM;
    const int KBall = (int)(K / kBK);
    const int kb0 = (int)((int64_t)split * KBall / splits), kb1 = (int)((int64_t)(split + 1) * KBall / splits);
    const int KB = kb1 - kb0;                                   // k-blocks of this CTA

    // ---------------------------------------------------------------- set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < SX; s++) {
            ptx::mbar_init(&bars->full_x[s], 1);
            ptx::mbar_init(&bars->empty_x[s], 1);
        }
        for (int s = 0; s < SA; s++) {
            ptx::mbar_init(&bars->full_a[s], kDequantWarps);
            ptx::mbar_init(&bars->empty_a[s], 1);
        }
        ptx::mbar_init(&bars->acc_full, 1);
        ptx::mbar_init(&bars->drain, 1);
        bars->abort = 0;
        bars->staged = 0;
        ptx::fence_barrier_init();
        ptx::tma_prefetch_desc(&tmap_x);
    }
    if (warp == 0) {
        ptx::tmem_alloc(&bars->tmem_base, C::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_d = bars->tmem_base;
    // The split-tail grid (and, after it, the reduce) reads only X and the weights, never this
    // grid's output, so it may start on each SM as soon as a CTA of this grid leaves it. The
    // whole-tile grid of a bf16-x call is itself a dependent of the conversion pass: there only
    // the TMA producer (which reads x16) and the epilogue (tok_fac) wait for that pass, and the
    // producer lets the split-tail grid launch only after its wait, so that grid, which never
    // waits for its own predecessor, also starts after the conversion. The dequant warps read
    // only the weights and start at once. (griddepcontrol.wait is a no-op for an ordinary
    // launch.)
    if (splits > 1)
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            if (splits == 1) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
            }
            int issued = 0;
            for (int kb = 0; kb < KB; kb++) {
                const int s = kb % SX;
                const uint32_t ph = (kb / SX) & 1;
                if (!ptx::mbar_wait_bounded_sleep(&bars->empty_x[s], ph ^ 1, abort, err, kDevErrTimeout, wait_ns))
                    break;
                ptx::mbar_arrive_expect_tx(&bars->full_x[s], C::kXBytes);
                ptx::tma_load_2d(xs + s * C::kXBytes, &tmap_x, &bars->full_x[s], (kb0 + kb) * kBK, (int32_t)m0);
                issued++;
            }
            // no copy may still be in flight when the CTA exits
            for (int kb = issued > SX ? issued - SX : 0; kb < issued; kb++) {
                volatile int no_abort = 0;
                ptx::mbar_wait_bounded(&bars->full_x[kb % SX], (kb / SX) & 1, &no_abort, err, kDevErrTimeout,
                                       kWaitLimitNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::umma_idesc_f16(0u, kBM, BN);   // fp16 x fp16 -> fp32
            int issued = 0;
            for (int kb = 0; kb < KB; kb++) {
                const int sx = kb % SX, sa = kb % SA;
                if (!ptx::mbar_wait_bounded(&bars->full_x[sx], (kb / SX) & 1, abort, err, kDevErrTimeout, wait_ns))
                    break;
                if (!ptx::mbar_wait_bounded(&bars->full_a[sa], (kb / SA) & 1, abort, err, kDevErrTimeout, wait_ns))
                    break;
                ptx::tc_fence_after();
                const uint32_t a_tmem = tmem_d + BN + 32 * sa;
                const uint64_t bdesc = ptx::sw128_kmajor_desc(ptx::smem_u32(xs + sx * C::kXBytes));
#pragma unroll
                for (int k = 0; k < kBK / 16; k++)   // K step k: 16 elements = 8 A columns, 32 B of the X rows
                    ptx::umma_f16_ts(tmem_d, a_tmem + 8 * k, bdesc + 2 * k, idesc, (kb | k) != 0);
                ptx::umma_commit(&bars->empty_x[sx]);   // both slots are free once these MMAs finish
                ptx::umma_commit(&bars->empty_a[sa]);
                issued++;
            }
            if (issued == KB) {
                ptx::umma_commit(&bars->acc_full);
            } else {
                // aborted: wait for the MMAs already issued before TMEM is released
                ptx::umma_commit(&bars->drain);
                volatile int no_abort = 0;
                ptx::mbar_wait_bounded(&bars->drain, 0, &no_abort, err, kDevErrTimeout, kWaitLimitNs);
            }
        }
    } else {
        // ------------------------------------------------------------ dequant, then epilogue
        // warp w = 2 + 4 h + j, lane l: row 32 (w % 4) + l of the tile (a warp reaches only its
        // own quarter of the tensor-memory lanes), half h of every k-block (chunks 4h .. 4h+3 of
        // 8 weights: one binary word or two ternary words)
        const int hk = (warp - 2) >> 2;                     // part of the k-block, 0 .. kParts-1
        const int r = 32 * (warp & 3) + lane;                // weight row within the tile
        const int64_t n = n0 + r;
        const bool row_ok = n < N;
        const int64_t G = K / 128;
        constexpr int kWts = kBK / kParts;                   // weights per thread per k-block
        constexpr int kCols = kWts / 2;                      // 32-bit TMEM columns per thread
        constexpr int kBitsPerW = FMT == BQ_BINARY_G128 ? 1 : 2;
        constexpr int WPT = (kWts * kBitsPerW + 31) / 32;    // words per thread per k-block (1 or 2)
        // the thread's first bit: word hk * kWts * bits / 32 of the k-block, shifted by the rest
        const int bitpos = hk * kWts * kBitsPerW;
        const int bshift = bitpos & 31;
        const uint32_t *wrow = words + (row_ok ? n : 0) * (K / 32 * kBitsPerW) + (bitpos >> 5);
        const uint16_t *srow = scales + (row_ok ? n : 0) * G;
        // this thread's row in tensor memory: lane r (the warp's lane quarter), columns 16 hk ..
        const uint32_t arow_tmem = tmem_d + ((uint32_t)(32 * (warp & 3)) << 16) + BN + kCols * hk;

        constexpr int kAhead = FMT == BQ_TERNARY_B3_G128 ? 8 : 4;   // k-blocks of packed weights loaded ahead
        uint2 wq[kAhead];
        uint16_t sq[kAhead];
        // base-3 rows: 26 G bytes each, an even number, so every 16-bit load below is aligned
        const uint8_t *brow = reinterpret_cast<const uint8_t *>(words) + (row_ok ? n : 0) * (b3::kGroupBytes * G);
        auto load_kb = [&](int kbl, uint2 &wv_, uint16_t &sv_) {   // kbl: k-block of this CTA
            const int kbg = kb0 + kbl;
            if (FMT == BQ_TERNARY_B3_G128) {
                const int64_t g = kbg >> 1, f = g & ~int64_t(7);
                const int64_t nb = G - f < 8 ? G - f : 8;
                const int V = 2 * (kbg & 1) + hk;
                const uint8_t *five = brow + b3::kGroupBytes * f + 24 * (g - f) + b3_pf_start(V);
                const uint8_t *four = brow + b3::kGroupBytes * f + 24 * nb + 2 * (g - f);
                const uint32_t h0 = __ldg(reinterpret_cast<const uint16_t *>(five));
                const uint32_t h1 = __ldg(reinterpret_cast<const uint16_t *>(five + 2));
                const uint32_t h2 = __ldg(reinterpret_cast<const uint16_t *>(five + 4));
                const uint32_t h3 = __ldg(reinterpret_cast<const uint16_t *>(V == 3 ? four : five + 6));
                wv_ = make_uint2(h0 | (h1 << 16), h2 | (h3 << 16));
            } else if (WPT == 1)
                wv_ = make_uint2(__ldg(wrow + (size_t)kbg * 2 * kBitsPerW) >> bshift, 0u);
            else
                wv_ = __ldg(reinterpret_cast<const uint2 *>(wrow + (size_t)kbg * 4));
            sv_ = __ldg(srow + kbg / 2);
        };
#pragma unroll
        for (int i = 0; i < kAhead; i++) {
            wq[i] = make_uint2(0, 0);
            sq[i] = 0;
            if (row_ok && i < KB)
                load_kb(i, wq[i], sq[i]);
        }
        for (int kb = 0; kb < KB; kb++) {
            const uint2 wv = wq[0];
            const uint16_t sv = sq[0];
#pragma unroll
            for (int i = 0; i < kAhead - 1; i++) {
                wq[i] = wq[i + 1];
                sq[i] = sq[i + 1];
            }
            const int nk = kb + kAhead;
            wq[kAhead - 1] = make_uint2(0, 0);
            if (row_ok && nk < KB)
                load_kb(nk, wq[kAhead - 1], sq[kAhead - 1]);

            const int s = kb % SA;
            const uint32_t ph = (kb / SA) & 1;
            if (!warp_wait(&bars->empty_a[s], ph ^ 1, abort, err, wait_ns))
                break;
            ptx::tc_fence_after();
            const uint32_t s2 = row_ok ? scale_pair(sv) : 0u;
            uint32_t av[kCols];                              // 2 weights per 32-bit column
            if constexpr (FMT == BQ_TERNARY_B3_G128) {
                static_assert(kCols == 16, "a base-3 part is 32 weights");
                switch (2 * ((kb0 + kb) & 1) + hk) {
                case 0: expand_pairs_b3<0>(wv, s2, av); break;
                case 1: expand_pairs_b3<1>(wv, s2, av); break;
                case 2: expand_pairs_b3<2>(wv, s2, av); break;
                default: expand_pairs_b3<3>(wv, s2, av); break;
                }
            } else {
                expand_pairs<FMT, kCols>(wv, s2, av);
            }
            if (!row_ok) {
#pragma unroll
                for (int c = 0; c < kCols; c++)
                    av[c] = 0u;
            }
            if constexpr (kCols == 16)
                ptx::tmem_st_32x32b_x16(arow_tmem + 32 * s, *reinterpret_cast<const uint32_t(*)[16]>(av));
            else
                ptx::tmem_st_32x32b_x8(arow_tmem + 32 * s, *reinterpret_cast<const uint32_t(*)[8]>(av));
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(&bars->full_a[s]);
        }

        // ------------------------------------------------------------ epilogue
        // Whole tiles whose output rows are 16-byte aligned go through shared memory (the X ring,
        // idle once the last MMA has completed) and leave as one TMA tile store: [BN tokens][128
        // rows] in the output type, clipped by the tensor map at M and N. Otherwise each warp
        // stores its 32-row segments directly; split tiles store fp32 partials.
        const bool staged_out = splits == 1 && y_tma;
        if (tok_fac && splits == 1)
            asm volatile("griddepcontrol.wait;" ::: "memory");   // tok_fac comes from the conversion pass
        if (warp_wait(&bars->acc_full, 0, abort, err, wait_ns)) {
            ptx::tc_fence_after();
            const int quad = warp & 3;                       // TMEM lanes 32*quad .. +31
            const int64_t nrow = n0 + quad * 32 + lane;
            const bool nok = nrow < N;
            // the kParts warps of a lane quarter take alternate 32-token column blocks
#pragma unroll 1
            for (int cc = hk; cc < BN / 32; cc += kParts) {
                uint32_t v[32];
                ptx::tmem_ld_32x32b_x32(tmem_d + ((uint32_t)(quad * 32) << 16) + cc * 32, v);
                ptx::tmem_wait_ld();
                const int64_t mbase = m0 + cc * 32;
                if (tok_fac && splits == 1) {
                    // undo the per-token power of two of bf16 x (exact); split partials are
                    // scaled by the reduce pass
#pragma unroll
                    for (int j = 0; j < 32; j++) {
                        const int64_t m = mbase + j < M ? mbase + j : M - 1;
                        v[j] = __float_as_uint(__uint_as_float(v[j]) * __ldg(tok_fac + m));
                    }
                }
                if (splits > 1) {
                    // fp32 partial of this split: [tail tile][split][BN tokens][128 rows]
                    float *pt = part + (((size_t)(tile - tile0) * splits + split) * BN + cc * 32) * kBM + quad * 32 + lane;
#pragma unroll
                    for (int j = 0; j < 32; j++)
                        pt[(size_t)j * kBM] = __uint_as_float(v[j]);
                    continue;
                }
                if (staged_out) {
                    const int e0 = (cc * 32) * kBM + quad * 32 + lane;   // token cc*32, this row
#pragma unroll
                    for (int j = 0; j < 32; j++) {
                        const float f = __uint_as_float(v[j]);
                        if (yt == BQ_F32)
                            store_out(reinterpret_cast<float *>(xs) + e0 + j * kBM, f);
                        else if (yt == BQ_BF16)
                            store_out(reinterpret_cast<__nv_bfloat16 *>(xs) + e0 + j * kBM, f);
                        else
                            store_out(reinterpret_cast<__half *>(xs) + e0 + j * kBM, f);
                    }
                    continue;
                }
                if (!nok)
                    continue;
#pragma unroll
                for (int j = 0; j < 32; j++) {
                    const int64_t m = mbase + j;
                    if (m < M) {
                        const float f = __uint_as_float(v[j]);
                        if (yt == BQ_F32)
                            store_out(static_cast<float *>(y) + m * N + nrow, f);
                        else if (yt == BQ_BF16)
                            store_out(static_cast<__nv_bfloat16 *>(y) + m * N + nrow, f);
                        else
                            store_out(static_cast<__half *>(y) + m * N + nrow, f);
                    }
                }
            }
            if (staged_out) {
                ptx::fence_proxy_async_smem();               // the tile store reads these writes
                __syncwarp();
                if (lane == 0)
                    atomicAdd(&bars->staged, 1);
            }
        }
        if (staged_out) {
            // every epilogue warp passes here once, whatever its waits returned
            asm volatile("bar.sync 1, %0;" ::"n"(kDequantWarps * 32) : "memory");
            if (threadIdx.x == 64 && *reinterpret_cast<volatile int *>(&bars->staged) == kDequantWarps) {
                ptx::tma_store_2d(&tmap_y, xs, (int32_t)n0, (int32_t)m0);
                ptx::bulk_commit_group();
                ptx::bulk_wait_all();
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_d, C::kTmemCols);
    }
    // launched as a dependent of the whole-tile grid, this grid completes only after that one
    // has, so work queued behind it on the stream sees both (a no-op for an ordinary launch)
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Y for the tiles that were split along K: the fp32 partials of each output added in split
// order (so the result does not depend on timing), then rounded once to the output type.
template <int BN>
__global__ void __launch_bounds__(256)
prefill_reduce_kernel(const float *__restrict__ part, int tiles, int splits, int tiles_m, int tile0, int64_t M,
                      int64_t N, void *__restrict__ y, int yt, const float *__restrict__ tok_fac)
{
    // launched as a dependent of the split grid: wait until that grid (and through it the
    // whole-tile grid) has completed and its partials are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t idx = (int64_t)blockIdx.x * 256 + threadIdx.x;   // (tail tile, token, row)
    if (idx >= (int64_t)tiles * BN * kBM)
        return;
    const int t = (int)(idx / (BN * kBM)), mr = (int)(idx % (BN * kBM));
    const int ml = mr / kBM, rl = mr % kBM;
    const int tile = tile0 + t;
    const int64_t m = (int64_t)(tile % tiles_m) * BN + ml, n = (int64_t)(tile / tiles_m) * kBM + rl;
    if (m >= M || n >= N)
        return;
    const float *p = part + (size_t)t * splits * BN * kBM + mr;
    float v = 0.f;
    for (int sp = 0; sp < splits; sp++)
        v += p[(size_t)sp * BN * kBM];
    if (tok_fac)
        v *= tok_fac[m];                                   // exact power of two (bf16 x)
    if (yt == BQ_F32)
        store_out(static_cast<float *>(y) + m * N + n, v);
    else if (yt == BQ_BF16)
        store_out(static_cast<__nv_bfloat16 *>(y) + m * N + n, v);
    else
        store_out(static_cast<__half *>(y) + m * N + n, v);
}

int sm_count_pf()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

// Tile schedule: whole waves of one tile per CTA; when the last wave would be short (at most
// half the SMs), its tiles are split along K over the idle SMs instead, and a reduce kernel
// adds the splits. M = 512, N = 20480 at BN = 256: 320 tiles = 2 waves of 148 + 24 tiles,
// which become 24 x 6 split CTAs instead of a third, mostly empty wave.
struct PfPlan {
    int tiles_m, tiles, full, tail, splits;
};

PfPlan pf_plan(int64_t M, int64_t N, int64_t K, int BN)
{
    PfPlan p;
    p.tiles_m = (int)((M + BN - 1) / BN);
    p.tiles = p.tiles_m * (int)((N + kBM - 1) / kBM);
    const int sms = sm_count_pf();
    const int waves = p.tiles / sms;
    p.tail = p.tiles - waves * sms;
    p.splits = 1;
    if (waves >= 1 && p.tail > 0 && p.tail <= sms / 2) {
        p.splits = sms / p.tail < 8 ? sms / p.tail : 8;
        const int kblocks = (int)(K / kBK);          // every split gets at least 4 k-blocks
        if (p.splits > kblocks / 4)
            p.splits = kblocks / 4;
        if (p.splits < 2)
            p.splits = 1;
    }
    if (p.splits == 1)
        p.tail = 0;
    p.full = p.tiles - p.tail;
    return p;
}

int bn_for(int64_t M) { return M <= 64 ? 64 : (M <= 128 ? 128 : 256); }

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
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

// Workspace: [fp32 partials of the split tail tiles][fp16 x16 [M][K]][tok_fac [M]], each
// 256-byte aligned. The x16 part serves bf16 x only; it is reserved for either x type so
// that the size does not depend on x's type.
struct PfWs {
    size_t part, x16, fac, total;
};

PfWs pf_ws(int64_t M, int64_t N, int64_t K)
{
    auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
    const int bn = bn_for(M);
    const PfPlan pl = pf_plan(M, N, K, bn);
    PfWs w;
    w.part = 0;
    w.x16 = al((size_t)pl.tail * pl.splits * bn * kBM * sizeof(float));
    w.fac = w.x16 + al((size_t)M * (size_t)K * 2);
    w.total = w.fac + al((size_t)M * sizeof(float));
    return w;
}

template <int FMT, int BN>
cudaError_t launch_t(const PrefillArgs &a, cudaStream_t s)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return cudaErrorNotSupported;
    const PfWs ws = pf_ws(a.M, a.N, a.K);
    uint8_t *wsb = static_cast<uint8_t *>(a.workspace);
    const bool bf16 = a.xt == BQ_BF16;
    const void *xop = bf16 ? static_cast<const void *>(wsb + ws.x16) : a.x;
    float *tok_fac = bf16 ? reinterpret_cast<float *>(wsb + ws.fac) : nullptr;
    CUtensorMap map;
    cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.M};
    cuuint64_t strides[1] = {(cuuint64_t)a.K * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)BN};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(xop), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // Y as [M][N] in the output type, stored in [BN tokens][128 rows] boxes; usable when a row
    // of Y is a whole number of 16-byte units (the tensor map's stride rule)
    CUtensorMap map_y;
    std::memset(&map_y, 0, sizeof(map_y));
    const int esize = a.yt == BQ_F32 ? 4 : 2;
    int y_tma = 0;
    if ((a.N * esize) % 16 == 0) {
        cuuint64_t ydims[2] = {(cuuint64_t)a.N, (cuuint64_t)a.M};
        cuuint64_t ystrides[1] = {(cuuint64_t)a.N * esize};
        cuuint32_t ybox[2] = {(cuuint32_t)kBM, (cuuint32_t)BN};
        const CUtensorMapDataType yd = a.yt == BQ_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                       : a.yt == BQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        y_tma = enc(&map_y, yd, 2, a.y, ydims, ystrides, ybox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    auto kern = prefill_kernel<FMT, BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<BN>::kSmem);
    if (e != cudaSuccess)
        return e;
    const PfPlan pl = pf_plan(a.M, a.N, a.K, BN);
    const uint16_t *sc = reinterpret_cast<const uint16_t *>(a.scales);
    float *part = reinterpret_cast<float *>(wsb + ws.part);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (bf16) {
        // conversion pass (an ordinary launch: x may be the previous kernel's output), then the
        // whole-tile grid as its programmatic dependent: the GEMM CTAs allocate tensor memory
        // and set up their barriers while the conversion runs, and wait for it in
        // griddepcontrol.wait
        prefill_x16_kernel<<<(unsigned)a.M, kX16Threads, 0, s>>>(static_cast<const __nv_bfloat16 *>(a.x), a.K,
                                                                 reinterpret_cast<__half *>(wsb + ws.x16), tok_fac);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
        cudaLaunchConfig_t wcfg = {};
        wcfg.gridDim = dim3((unsigned)pl.full);
        wcfg.blockDim = dim3(kThreads);
        wcfg.dynamicSmemBytes = Cfg<BN>::kSmem;
        wcfg.stream = s;
        wcfg.attrs = attr;
        wcfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&wcfg, kern, map, map_y, y_tma, a.words, sc, a.M, a.N, a.K, a.y, a.yt, pl.tiles_m, 0,
                               1, part, (const float *)tok_fac, a.dev_status, a.wait_ns);
    } else {
        kern<<<pl.full, kThreads, Cfg<BN>::kSmem, s>>>(map, map_y, y_tma, a.words, sc, a.M, a.N, a.K, a.y, a.yt,
                                                       pl.tiles_m, 0, 1, part, (const float *)nullptr, a.dev_status,
                                                       a.wait_ns);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess)
        return e;
    if (pl.tail > 0) {
        // programmatic dependent launches: the tail CTAs take the SMs the whole-tile grid
        // frees without waiting for all of it (the whole-tile grid lets them launch only after
        // its own predecessors, including the conversion pass, are complete), and the reduce is
        // resident before the tail grid ends, waiting on it in griddepcontrol.wait
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(pl.tail * pl.splits));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = Cfg<BN>::kSmem;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, map, map_y, y_tma, a.words, sc, a.M, a.N, a.K, a.y, a.yt, pl.tiles_m,
                               pl.full, pl.splits, part, (const float *)tok_fac, a.dev_status, a.wait_ns);
        if (e != cudaSuccess)
            return e;
        const int64_t n_out = (int64_t)pl.tail * BN * kBM;
        cudaLaunchConfig_t rcfg = {};
        rcfg.gridDim = dim3((unsigned)((n_out + 255) / 256));
        rcfg.blockDim = dim3(256);
        rcfg.stream = s;
        rcfg.attrs = attr;
        rcfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&rcfg, prefill_reduce_kernel<BN>, (const float *)part, pl.tail, pl.splits, pl.tiles_m,
                               pl.full, a.M, a.N, a.y, a.yt, (const float *)tok_fac);
        if (e != cudaSuccess)
            return e;
    }
    return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_bn(const PrefillArgs &a, cudaStream_t s)
{
    const int bn = bn_for(a.M);
    if (bn == 64)
        return launch_t<FMT, 64>(a, s);
    if (bn == 128)
        return launch_t<FMT, 128>(a, s);
    return launch_t<FMT, 256>(a, s);
}

}  // namespace

// fp32 partials of the split tail tiles (none when the tiles fill whole waves or the last wave
// is more than half full), the fp16 copy of bf16 x and its per-token factors
size_t prefill_workspace_bytes(int64_t M, int fmt, int64_t N, int64_t K)
{
    (void)fmt;
    return pf_ws(M, N, K).total;
}

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t s, unsigned *launches)
{
    *launches = (pf_plan(a.M, a.N, a.K, bn_for(a.M)).tail > 0 ? 3 : 1) + (a.xt == BQ_BF16 ? 1 : 0);
    if (a.fmt == BQ_BINARY_G128)
        return launch_bn<BQ_BINARY_G128>(a, s);
    if (a.fmt == BQ_TERNARY_B3_G128)
        return launch_bn<BQ_TERNARY_B3_G128>(a, s);
    return launch_bn<BQ_TERNARY_G128>(a, s);
}

}  // namespace bq
