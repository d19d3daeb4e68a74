// gemv_rows.cu -- decode GEMV (M <= 8 token rows) on packed binary-g128 / ternary-g128 weights,
// every CTA owning whole output rows (all of K).
//
// Model card "prism-ml/Bonsai-27B-mlx-1bit", sections "Weight representation: Binary g128" and
// "CUDA (NVIDIA GPUs)": y[m][n] = sum_g s[n][g] * sum_{k in g} v[n][k] x[m][k], v = +-1 (binary)
// or {-1, 0, +1} (ternary: "Ternary Bonsai 27B vs ..." article, wmrh.cn); the packed weights are
// unpacked inside the product and each group scale is applied once per group. Batch-1 decode
// (tg128) is the memory-bound phase of section "Cross-platform throughput", and on H100 the
// pages found it bound by launch and synchronisation latency rather than by bandwidth; this
// kernel is shaped by both.
//
// The arithmetic is that of gemv_mma.cuh (sign bits as s8 operands of mma.sync m16n8k32, x as
// balanced integer digits, exact int32 column sums, the group scale once per group in fp32).
// Why mma.sync and not tcgen05 here: a kind::i8 tcgen05.mma with the sign operand in tensor
// memory measured at least ~44 cycles per instruction at N <= 64 (a 128 x 32 tile, ~93
// weights per SM clock) and tcgen05.st of the expanded operand ~78 bytes per SM clock, both
// below the ~160 binary weights per SM clock that HBM delivers; mma.sync takes its operands from
// registers and peaks at ~240.
//
// Every wait is bounded: a pipeline wait that gives up (after 2 s, or the shorter test limit of
// bq_debug_set_wait_limit_ns) records kDevErrTimeout and makes the CTA skip its remaining work;
// the producer still waits (2 s at most) for its copies in flight before the CTA exits.
//
// What this file decides is the work split and the latency of a call:
//   * Rows. The N outputs are 16-row tiles; CTA b owns tiles [b T / P, (b+1) T / P) over all of
//     K, so no output is split between CTAs: no partial sums in device memory, no counters, no
//     finalize pass. (A K-split between CTAs cost about 2 us of every small call: partial
//     stores, an atomic and dependent loads from L2 by the last CTA.)
//   * Warps. A warp group's 8 consumer warps take the 8 groups of a 1024-k slice, one each, for
//     up to 4 tiles of a tile-group: a warp loads the x fragment of its group once and uses it
//     for all its tiles. With 16 consumer warps (one column set, long streams) the second warp
//     group takes tiles 4..7. After the last slice of a tile-group the eight per-group sums of
//     each output meet in shared memory and are added in group order (deterministic).
//   * Weights. A producer lane streams, per (tile-group, slice), one TMA box of 16 rows x 128
//     bytes of packed words per tile (two for ternary) and one box of the 16 rows' 8 group
//     scales, into a ring of stages; only whole tiles of the CTA are loaded. The producer never
//     waits for the previous kernel: the weights do not depend on it, so a CTA that becomes
//     resident early (programmatic dependent launch) prefetches its first stages meanwhile.
//   * x. A prep kernel turns x into the digit fragments of every (group, token) once per call
//     (one warp each, in parallel over the GPU) and every CTA copies them in with one bulk copy.
//     Building them inside each CTA measured slower: a CTA's 8 warps took several microseconds
//     for the chains of warp-wide reductions of 40 to 320 items.
#include <cuda.h>

#include <mutex>

#include "bq_internal.cuh"
#include "gemv_mma.cuh"
#include "sm100_ptx.cuh"
#include "topk.cuh"

namespace bq {
namespace {

using namespace mma8;

constexpr int kGroupWarps = 8;                // warps of a warp group: one per group of a 1024-k slice
constexpr int kWarpTiles = 4;                 // 16-row tiles a warp takes per slice
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 227 * 1024;
constexpr int kSmemPair = 113 * 1024;         // two CTAs fit on one SM below this
constexpr uint64_t kWaitLimitNs = kWaitLimitDefaultNs;   // drain waits before exit

template <int FMT> struct RCfg {
    static constexpr bool kB3 = FMT == BQ_TERNARY_B3_G128;
    static constexpr int kBoxes = FMT == BQ_TERNARY_G128 ? 2 : 1;      // boxes per tile per slice
    static constexpr int kBoxInner = kB3 ? b3::kBlockBytes : 32;      // box width: 208 bytes or 32 words
    static constexpr int kBoxBytes = 16 * (kB3 ? b3::kBlockBytes : 128);
    static constexpr int kTileBytes = kBoxBytes * kBoxes;             // packed weights of a tile per slice
};

struct RLayout {
    int frag, colf, cfix, red, lg, tks, tko, ring, bars, total, stage_bytes, scale_off;
};

// Shared-memory layout (host and device compute the same thing). topk adds the selection scratch
// and its k output keys, lg_floats the CTA's logits [M][rows] (when they are kept on chip).
template <int FMT, int CS>
__host__ __device__ inline RLayout rows_layout(int G, int TB, int S, int lg_floats = 0, bool topk = false)
{
    RLayout L;
    L.frag = 0;                                           // [CS][G][2][32][4] u32
    L.colf = CS * G * 1024;                               // [2 CS][G] f32
    L.cfix = L.colf + 2 * CS * G * 4;                     // [CS][G][8] s32
    L.red = L.cfix + CS * G * 32;                         // [2][8 groups][TB][CS][16 rows][2] f32
    L.lg = L.red + 2 * kGroupWarps * TB * CS * 32 * 4;    // top-k: [M][rows] f32
    L.tks = (L.lg + 4 * lg_floats + 15) / 16 * 16;        // top-k: selection scratch
    L.tko = L.tks + (topk ? (int)sizeof(topk::Smem) : 0);        // top-k: k output keys
    L.ring = (L.tko + (topk ? 8 * topk::kMaxK : 0) + 1023) / 1024 * 1024;
    L.scale_off = TB * RCfg<FMT>::kTileBytes;             // scales [TB][16 rows][8] fp16 after the words
    L.stage_bytes = (L.scale_off + TB * 256 + 1023) / 1024 * 1024;
    L.bars = L.ring + S * L.stage_bytes;
    L.total = L.bars + 2 * kMaxStages * 8 + 8 + 16 + 1024;   // barriers, abort flag, alignment slack
    return L;
}

struct Bars {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t frag;
    int abort;
};

// Digit fragments of every (group, token) of x, once per call: one warp per (group, token);
// slots of the last column set past M are left as they are (their columns are never stored).
template <int FMT, int CS, typename XT>
__global__ void __launch_bounds__(256)
gemv_rows_prep_kernel(const XT *__restrict__ x, int M, int64_t K, uint32_t *__restrict__ frag,
                      float *__restrict__ colf, int *__restrict__ cfix, unsigned int *__restrict__ topk_counter)
{
    // the GEMV that reads these fragments may set itself up and stream its weights meanwhile
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // x may be the previous kernel's output, and the previous GEMV may still read the workspace
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int G = (int)(K / 128);
    const int item = (int)((blockIdx.x * 256 + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (topk_counter && blockIdx.x == 0 && threadIdx.x == 0)
        *topk_counter = 0u;                      // the top-k ticket of the GEMV that follows
    if (item < G * M) {
        if (FMT == BQ_TERNARY_B3_G128)
            build_item_b3<CS, XT>(x, M, K, G, item, lane, frag, colf, cfix);
        else
            build_items<FMT, CS, XT, 1>(x, M, K, G, item, 1, lane, frag, colf, cfix);
    }
}

// Per-thread constants of the inner loop.
struct Lane {
    uint32_t mul[9];                  // shift multipliers and byte masks of the sign expansion
    int off0, off1, soff0, soff1;     // byte offsets of this thread's words / scales in a tile
    int offh, offt;                   // base-3: its two-byte half and four-code byte (row g8)
    uint32_t mt;                      // base-3: 3^l1 + 2^16 3^l2, the levels of its four-code byte
};

// Base-3: the A operands of one group for this thread's rows g8 and g8 + 8 of a tile (rows are
// 208 bytes apart in shared memory), in the register order of expand_group.
__device__ __forceinline__ void expand_group_b3(const uint8_t *wt, const Lane &ln, uint32_t (&quad)[4][4])
{
    constexpr int kRow8 = 8 * b3::kBlockBytes;
    uint32_t a0[8], a1[8];
    expand_b3(*reinterpret_cast<const uint32_t *>(wt + ln.off0), *reinterpret_cast<const uint16_t *>(wt + ln.offh),
              wt[ln.offt], ln.mt, a0);
    expand_b3(*reinterpret_cast<const uint32_t *>(wt + ln.off0 + kRow8),
              *reinterpret_cast<const uint16_t *>(wt + ln.offh + kRow8), wt[ln.offt + kRow8], ln.mt, a1);
#pragma unroll
    for (int j = 0; j < 4; j++) {
        quad[j][0] = a0[2 * j];
        quad[j][1] = a1[2 * j];
        quad[j][2] = a0[2 * j + 1];
        quad[j][3] = a1[2 * j + 1];
    }
}

// One slice (1024 k) of NTL tiles j0, j0 + WG, j0 + 2 WG, ... of the stage, for the warp's
// group q: the x fragment, factors and accumulator inputs are loaded once, the tiles are
// expanded and multiplied two at a time at one or two column sets (two independent MMA chains).
// NTL is known at compile time, so a full tile-group runs without a branch.
template <int FMT, int CS, int WG, int NTL>
__device__ __forceinline__ void slice_tiles(const uint8_t *__restrict__ st, int j0, const Lane &ln,
                                            const uint32_t *__restrict__ frag_lane, const float *__restrict__ colf_tok,
                                            const int *__restrict__ cfix_t, int G, int q, int magic_in,
                                            float (&acc)[kWarpTiles][CS][4])
{
    using SCH = Scheme<FMT, CS>;
    constexpr int kTileBytes = RCfg<FMT>::kTileBytes;
    uint4 bA[CS], bB[CS];
    float f[CS];
    int2 cin2[CS];
#pragma unroll
    for (int cs = 0; cs < CS; cs++) {
        const uint32_t *fq = frag_lane + (size_t)(cs * G + q) * 256;
        bA[cs] = *reinterpret_cast<const uint4 *>(fq);
        bB[cs] = *reinterpret_cast<const uint4 *>(fq + 128);
        f[cs] = colf_tok[2 * cs * G + q];
        if (SCH::kColFix)
            cin2[cs] = *reinterpret_cast<const int2 *>(cfix_t + (cs * G + q) * 8);
    }
    const int magic[4] = {magic_in, magic_in, magic_in, magic_in};   // constant accumulator input (not kMask)
    // two tiles at a time at one or two column sets; one at a time beyond, where the column sets
    // already give independent MMA chains and the accumulators fill the registers
    constexpr int kPair = CS <= 2 ? 2 : 1;
#pragma unroll
    for (int jl = 0; jl < NTL; jl += kPair) {
        const int np = NTL - jl < kPair ? NTL - jl : kPair;   // tiles in this step (compile time after unrolling)
        uint32_t A[2][4][4];
        float s0[2], s1[2];
#pragma unroll
        for (int h = 0; h < 2; h++) {
            if (h < np) {
                const int j = j0 + (jl + h) * WG;              // tile of the stage
                const uint8_t *wt = st + j * kTileBytes;
                if (SCH::kB3)
                    expand_group_b3(wt, ln, A[h]);
                else
                    expand_group<FMT, SCH::kMask>(wt + ln.off0, wt + ln.off1, ln.mul, A[h]);
                const uint8_t *sp = st + j * 256;
                s0[h] = __half2float(*reinterpret_cast<const __half *>(sp + ln.soff0));
                s1[h] = __half2float(*reinterpret_cast<const __half *>(sp + ln.soff1));
            }
        }
#pragma unroll
        for (int cs = 0; cs < CS; cs++) {
            int d[2][4];
#pragma unroll
            for (int h = 0; h < 2; h++) {
                if (h < np) {
                    constexpr bool U8 = SCH::kB3;
                    if (SCH::kColFix) {
                        const int cin[4] = {cin2[cs].x, cin2[cs].y, cin2[cs].x, cin2[cs].y};
                        mma_i8_first<U8>(d[h], A[h][0][0], A[h][0][1], A[h][0][2], A[h][0][3], bA[cs].x, bA[cs].y, cin);
                    } else {
                        mma_i8_first<U8>(d[h], A[h][0][0], A[h][0][1], A[h][0][2], A[h][0][3], bA[cs].x, bA[cs].y,
                                         magic);
                    }
                    mma_i8<U8>(d[h], A[h][1][0], A[h][1][1], A[h][1][2], A[h][1][3], bA[cs].z, bA[cs].w);
                    mma_i8<U8>(d[h], A[h][2][0], A[h][2][1], A[h][2][2], A[h][2][3], bB[cs].x, bB[cs].y);
                    mma_i8<U8>(d[h], A[h][3][0], A[h][3][1], A[h][3][2], A[h][3][3], bB[cs].z, bB[cs].w);
                }
            }
#pragma unroll
            for (int h = 0; h < 2; h++) {
                if (h < np) {
                    // the group scales of rows g8, g8 + 8 times this token's 2^(e-27)
                    const float sf0 = s0[h] * f[cs], sf1 = s1[h] * f[cs];
                    // exact int -> float: the accumulator started at the bits of 1.5 * 2^23
                    float *a = acc[jl + h][cs];
                    a[0] = fmaf(__int_as_float(d[h][0]) - 12582912.f, sf0, a[0]);
                    a[1] = fmaf(__int_as_float(d[h][1]) - 12582912.f, sf0, a[1]);
                    a[2] = fmaf(__int_as_float(d[h][2]) - 12582912.f, sf1, a[2]);
                    a[3] = fmaf(__int_as_float(d[h][3]) - 12582912.f, sf1, a[3]);
                }
            }
        }
    }
}

// Top-k mode: instead of y, the k largest logits of every token (keys as in topk.cuh). Each CTA
// keeps its rows' logits in shared memory, selects their k largest and writes them to cand; the
// last CTA to finish (a ticket on counter, which the prep kernel zeroes) selects the k largest of
// all CTAs' candidates, writes vals / idx and, with u given, draws a token per row.
struct TopkParams {
    int k, lg_rows;                 // k <= 32; rows of the per-CTA logits buffer
    float *lg_glob;                 // the logits buffers [grid][M][lg_rows] in the workspace, or null
                                    // (kept in shared memory)
    unsigned long long *cand;       // [grid][M][k], then the k-th key of each [grid][M]
    unsigned int *counter;
    float *vals;                    // [M][k]
    int *idx;                       // [M][k]
    const float *u;                 // [M] uniform numbers, or null (no draw)
    float temp, top_p;
    int *tokens;                    // [M]
};

// The end of a top-k call, run by the NT consumer threads once their tile-groups are done.
template <int NT>
__device__ void topk_tail(const TopkParams &tp, const float *lg, topk::Smem *sm, unsigned long long *out, int M,
                          int64_t N, int t0, int t1, bool ok, unsigned long long *stage, int stage_bytes)
{
    const int tid = threadIdx.x;
    const int64_t row0 = (int64_t)t0 * 16;
    const int64_t rows_end = (int64_t)t1 * 16 < N ? (int64_t)t1 * 16 : N;
    const int nrow = (int)(rows_end - row0);                       // this CTA's rows (>= 1)
    const int kk = nrow < tp.k ? nrow : tp.k;
    asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");          // every logit is in lg
    for (int m = 0; m < M; m++) {
        const float *lm = lg + m * tp.lg_rows;
        topk::select<NT>([&](int i) { return topk::key_of(lm[i], (uint32_t)(row0 + i)); }, nrow, kk, sm, out, tid, 1);
        if (tid < tp.k) {
            // rows past the CTA's own (fewer than k) and aborted calls leave the lowest key
            const unsigned long long key = ok && tid < kk ? out[tid] : 0ull;
            tp.cand[((int64_t)blockIdx.x * M + m) * tp.k + tid] = key;
            if (tid == tp.k - 1)        // this CTA's k-th key: the k largest overall are all >= it
                tp.cand[(int64_t)gridDim.x * M * tp.k + (int64_t)blockIdx.x * M + m] = key;
        }
    }
    // ticket: the last CTA to arrive merges
    asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
    if (tid == 0) {
        __threadfence();
        sm->last = atomicAdd(tp.counter, 1u) == gridDim.x - 1;
        for (int m = 0; m < 8; m++)
            sm->floor[m] = 0ull;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
    if (!sm->last)
        return;
    __threadfence();
    const int n = (int)gridDim.x * tp.k;
    // The stage ring is idle now (every copy into it has been consumed): the candidates of a row go
    // there once. The k largest overall are all at or above the largest of the CTAs' k-th keys, so
    // only the candidates at or above that floor (usually a few more than k) need ranking.
    const bool staged = n * 8 <= stage_bytes;
    for (int m = 0; m < M; m++) {
        const unsigned long long *cm = tp.cand;
        const unsigned long long *kth = tp.cand + (int64_t)gridDim.x * M * tp.k;
        unsigned long long lo = 0ull;
        for (int c = tid; c < (int)gridDim.x; c += NT) {
            const unsigned long long v = __ldcg(kth + (int64_t)c * M + m);
            lo = v > lo ? v : lo;
        }
        if (staged)
            for (int i = tid; i < n; i += NT) {
                const int c = i / tp.k, j = i - c * tp.k;
                stage[i] = __ldcg(cm + ((int64_t)c * M + m) * tp.k + j);
            }
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, lo, d);
            lo = o > lo ? o : lo;
        }
        if ((tid & 31) == 0)
            atomicMax(&sm->floor[m], lo);
        if (tid == 0)
            sm->cnt = 0;
        asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
        lo = sm->floor[m];
        auto key_at = [&](int i) {
            if (staged)
                return stage[i];
            const int c = i / tp.k, j = i - c * tp.k;
            return __ldcg(cm + ((int64_t)c * M + m) * tp.k + j);
        };
        for (int i = tid; i < n; i += NT) {
            const unsigned long long key = key_at(i);
            if (key >= lo) {
                const int slot = atomicAdd(&sm->cnt, 1);
                if (slot < topk::kGather)
                    sm->buf[slot] = key;
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
        const int cnt = sm->cnt;
        if (cnt <= topk::kGather) {
            // rank = the number of larger keys (keys are unique)
            if (tid < cnt) {
                const unsigned long long a = sm->buf[tid];
                int r = 0;
                for (int j = 0; j < cnt; j++)
                    r += sm->buf[j] > a;
                if (r < tp.k)
                    out[r] = a;
            }
            asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
        } else {
            // many candidates tie near the floor: the radix selection over all of them
            topk::select<NT>(key_at, n, tp.k, sm, out, tid, 1);
        }
        if (tid < tp.k) {
            tp.vals[m * tp.k + tid] = topk::value_of(out[tid]);
            tp.idx[m * tp.k + tid] = (int)topk::index_of(out[tid]);
        }
        if (tp.u && tid < 32) {
            const int tok = topk::draw(out, tp.k, tp.temp, tp.top_p, tp.u[m], tid);
            if (tid == 0)
                tp.tokens[m] = tok;
        }
    }
    if (tid == 0)
        *tp.counter = 0u;
}

// Modes of the row kernel: the plain GEMV, the top-k selection, and the gate/up projection of a
// SwiGLU MLP (GLU): logical tile 2i is gate rows 16i .. 16i+15 (tmap_w, tmap_s), tile 2i+1 the
// same rows of up (tmap_w2, tmap_s2); CTAs and tile-groups hold whole pairs, and the epilogue
// writes y[m][n] = silu(gate) * up with silu(z) = z / (1 + e^-z) (N = the gate rows).
enum { kModePlain = 0, kModeTopk = 1, kModeGlu = 2 };

// WG warp groups of 8 consumer warps (WG = 2 only at one column set, for long streams): warp
// w takes group w % 8 of every slice and tiles w / 8, w / 8 + WG, ... of the tile-group.
template <int FMT, int CS, int WG, int MODE>
__global__ void __launch_bounds__((WG * kGroupWarps + 1) * 32, CS == 1 && WG == 1 ? 2 : 1)
gemv_rows_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_s,
                 const __grid_constant__ CUtensorMap tmap_w2, const __grid_constant__ CUtensorMap tmap_s2, int M,
                 int64_t N, int64_t K, void *__restrict__ y, int yt, int T, int TB, int S,
                 const uint32_t *__restrict__ frag_g, const float *__restrict__ colf_g, const int *__restrict__ cfix_g,
                 uint32_t one, unsigned int *dev_status, uint64_t wait_ns, const TopkParams tp)
{
    constexpr bool TOPK = MODE == kModeTopk, GLU = MODE == kModeGlu;
    using SCH = Scheme<FMT, CS>;
    constexpr int kConsumers = WG * kGroupWarps;
    constexpr int kTileBytes = RCfg<FMT>::kTileBytes, kBoxes = RCfg<FMT>::kBoxes;
    const int G = (int)(K / 128), C = (int)(K / 1024);
    const RLayout L = rows_layout<FMT, CS>(G, TB, S, TOPK && !tp.lg_glob ? M * tp.lg_rows : 0, TOPK);
    extern __shared__ uint8_t smem_raw[];
    // align by an offset on the shared array itself, so every access stays a shared-memory one
    uint8_t *smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    float *const lgp = TOPK ? (tp.lg_glob ? tp.lg_glob + (int64_t)blockIdx.x * M * tp.lg_rows
                                          : reinterpret_cast<float *>(smem + L.lg))
                            : nullptr;
    uint32_t *frag_s = reinterpret_cast<uint32_t *>(smem + L.frag);
    float *colf_s = reinterpret_cast<float *>(smem + L.colf);
    int *cfix_s = reinterpret_cast<int *>(smem + L.cfix);
    float *red = reinterpret_cast<float *>(smem + L.red);
    uint8_t *ring = smem + L.ring;
    Bars *bars = reinterpret_cast<Bars *>(smem + L.bars);
    volatile int *abort = &bars->abort;
    unsigned int *err = dev_status + kSlotErrBits;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = (int)gridDim.x;
    // whole tiles, or (GLU) whole gate/up pairs, per CTA
    const int t0 = GLU ? 2 * (int)((int64_t)blockIdx.x * (T / 2) / P) : (int)((int64_t)blockIdx.x * T / P);
    const int t1 = GLU ? 2 * (int)(((int64_t)blockIdx.x + 1) * (T / 2) / P) : (int)(((int64_t)blockIdx.x + 1) * T / P);
    const int ntg = (t1 - t0 + TB - 1) / TB;               // tile-groups of this CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            ptx::mbar_init(&bars->full[s], 1);
            ptx::mbar_init(&bars->empty[s], kConsumers);
        }
        ptx::mbar_init(&bars->frag, 1);
        bars->abort = 0;
        ptx::fence_barrier_init();
    }
    __syncthreads();
    // the next kernel in the stream may launch now; it waits for this grid before it reads
    // anything this grid writes
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == kConsumers) {
        // ------------------------------------------------------------------- producer
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tmap_w);
            ptx::tma_prefetch_desc(&tmap_s);
            if (GLU) {
                ptx::tma_prefetch_desc(&tmap_w2);
                ptx::tma_prefetch_desc(&tmap_s2);
            }
            int s = 0, it = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tg = 0; ok && tg < ntg; tg++) {
                const int tb = t0 + tg * TB;
                const int nt = t1 - tb < TB ? t1 - tb : TB;
                for (int c = 0; c < C; c++, it++) {
                    // a free slot: the producer sleeps in the wait, leaving the issue slots to the consumers
                    if (!ptx::mbar_wait_bounded_sleep(&bars->empty[s], ph ^ 1, abort, err, kDevErrTimeout,
                                                      wait_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = ring + s * L.stage_bytes;
                    ptx::mbar_arrive_expect_tx(&bars->full[s], (uint32_t)(nt * (kTileBytes + 256)));
                    for (int j = 0; j < nt; j++) {
                        const bool up = GLU && ((tb + j) & 1);
                        const int32_t row = (GLU ? (tb + j) >> 1 : tb + j) * 16;
                        const CUtensorMap *mw = up ? &tmap_w2 : &tmap_w;
                        const CUtensorMap *ms = up ? &tmap_s2 : &tmap_s;
#pragma unroll
                        for (int h = 0; h < kBoxes; h++)
                            ptx::tma_load_2d(st + j * kTileBytes + h * RCfg<FMT>::kBoxBytes, mw, &bars->full[s],
                                             (c * kBoxes + h) * RCfg<FMT>::kBoxInner, row);
                        ptx::tma_load_2d(st + L.scale_off + j * 256, ms, &bars->full[s], c * 8, row);
                    }
                    if (++s == S) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            // no copy may still be in flight when the CTA exits
            for (int k = it > S ? it - S : 0; k < it; k++) {
                volatile int no_abort = 0;
                ptx::mbar_wait_bounded(&bars->full[k % S], (uint32_t)((k / S) & 1), &no_abort, err, kDevErrTimeout,
                                       kWaitLimitNs);
            }
        }
    } else {
        // ------------------------------------------------------------------- consumers
        // the fragments come from the prep kernel launched just before this one
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const int w = warp & (kGroupWarps - 1), jb = warp / kGroupWarps;   // first tile of this warp
        const int g8 = lane >> 2, t = lane & 3;
        if (threadIdx.x == 0) {
            const uint32_t fb = (uint32_t)(CS * G * 1024), cb = (uint32_t)(2 * CS * G * 4), xb = (uint32_t)(CS * G * 32);
            ptx::mbar_arrive_expect_tx(&bars->frag, fb + cb + xb);
            ptx::bulk_load(frag_s, frag_g, fb, &bars->frag);
            ptx::bulk_load(colf_s, colf_g, cb, &bars->frag);
            ptx::bulk_load(cfix_s, cfix_g, xb, &bars->frag);
        }
        bool ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&bars->frag, 0, abort, err, kDevErrTimeout,
                                                                 wait_ns));

        Lane ln;
        if (SCH::kMask) {
            ln.mul[0] = one * 8u;
            ln.mul[1] = one * 64u;
            ln.mul[2] = one * 0x20202020u;
            ln.mul[3] = one * 0x40404040u;
            ln.mul[4] = one * 0x80808080u;
            ln.mul[5] = ln.mul[6] = ln.mul[7] = ln.mul[8] = 0u;
        } else {
#pragma unroll
            for (int i = 0; i < 7; i++)
                ln.mul[i] = one << (7 - i);
            ln.mul[7] = one * 0x80808080u;
            ln.mul[8] = one * 0x40404040u;
        }
        const int magic_in = (int)(one - 1u) + kMagic;
        // byte offsets, within a tile's words, of this thread's packed word(s) of group w in rows
        // g8 and g8 + 8 (128-byte rows, 128B swizzle: 16-byte chunk j of row r sits at j ^ (r & 7));
        // ternary groups 4..7 are in the tile's second box
        const int chunk = FMT == BQ_BINARY_G128 ? w : 2 * (w & 3) + (t >> 1);
        const int within = FMT == BQ_BINARY_G128 ? 4 * t : 8 * (t & 1);
        ln.off0 = (FMT == BQ_BINARY_G128 ? 0 : (w >> 2) * 2048) + g8 * 128 + ((chunk ^ g8) << 4) + within;
        ln.off1 = ln.off0 + 8 * 128;
        ln.offh = ln.offt = 0;
        ln.mt = 0u;
        if (SCH::kB3) {
            // 208-byte rows, no swizzle: five-code bytes of group w at 24 w, their thread's word at
            // + 4t and two-byte half at + 16 + 2t; the four-code bytes of group w at 192 + 2 w
            ln.off0 = g8 * b3::kBlockBytes + 24 * w + 4 * t;
            ln.off1 = ln.off0 + 8 * b3::kBlockBytes;
            ln.offh = g8 * b3::kBlockBytes + 24 * w + 16 + 2 * t;
            ln.offt = g8 * b3::kBlockBytes + 192 + 2 * w + (t >> 1);
            ln.mt = (t & 1) ? one * (27u + (81u << 16)) : one * (3u + (9u << 16));
        }
        ln.soff0 = L.scale_off + g8 * 16 + 2 * w;
        ln.soff1 = ln.soff0 + 8 * 16;
        const uint32_t *frag_lane = frag_s + lane * 4;
        const float *colf_tok = colf_s + (t >> 1) * G;
        const int *cfix_t = cfix_s + 2 * t;
        constexpr float kIn = SCH::kMask ? 64.f : 256.f;      // weight of the odd digit of a column pair
        const float hi = (t & 1) ? kIn * kIn : 1.f;           // columns 2t, 2t+1 are digits 2(t&1), +1

        int s = 0;
        uint32_t ph = 0;
        for (int tg = 0; tg < ntg; tg++) {
            const int tb = t0 + tg * TB;
            const int nt = t1 - tb < TB ? t1 - tb : TB;
            // this warp's tiles of the group: jb, jb + WG, ... (ntl of them)
            const int ntl = nt > jb ? (nt - jb + WG - 1) / WG : 0;
            float acc[kWarpTiles][CS][4];
#pragma unroll
            for (int j = 0; j < kWarpTiles; j++)
#pragma unroll
                for (int cs = 0; cs < CS; cs++)
#pragma unroll
                    for (int i = 0; i < 4; i++)
                        acc[j][cs][i] = 0.f;
            for (int c = 0; c < C; c++) {
                if (ok)
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&bars->full[s], ph, abort, err,
                                                                        kDevErrTimeout, wait_ns));
                if (ok) {
                    const uint8_t *st = ring + s * L.stage_bytes;
                    const int q = 8 * c + w;                    // this warp's group
                    switch (ntl) {                              // warp-uniform
                    case 4: slice_tiles<FMT, CS, WG, 4>(st, jb, ln, frag_lane, colf_tok, cfix_t, G, q, magic_in, acc); break;
                    case 3: slice_tiles<FMT, CS, WG, 3>(st, jb, ln, frag_lane, colf_tok, cfix_t, G, q, magic_in, acc); break;
                    case 2: slice_tiles<FMT, CS, WG, 2>(st, jb, ln, frag_lane, colf_tok, cfix_t, G, q, magic_in, acc); break;
                    case 1: slice_tiles<FMT, CS, WG, 1>(st, jb, ln, frag_lane, colf_tok, cfix_t, G, q, magic_in, acc); break;
                    default: break;
                    }
                }
                __syncwarp();
                if (lane == 0)
                    ptx::mbar_arrive(&bars->empty[s]);             // the stage's words are used up
                if (++s == S) {
                    s = 0;
                    ph ^= 1;
                }
            }

            // ---- the tile-group's outputs: each warp combines the digit columns of a token
            // (held by quad-threads t and t ^ 1), leaves its sums in shared memory, and after one
            // barrier the eight groups' sums of every output are added in group order
            float *rb = red + (tg & 1) * (kGroupWarps * TB * CS * 32);
#pragma unroll
            for (int jl = 0; jl < kWarpTiles; jl++) {
                const int j = jb + jl * WG;
                if (jl < ntl) {
#pragma unroll
                    for (int cs = 0; cs < CS; cs++) {
                        float v0 = fmaf(acc[jl][cs][1], kIn, acc[jl][cs][0]) * hi;   // row g8
                        float v1 = fmaf(acc[jl][cs][3], kIn, acc[jl][cs][2]) * hi;   // row g8 + 8
                        v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
                        v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
                        if ((t & 1) == 0) {
                            float *o = rb + ((w * TB + j) * CS + cs) * 32 + (t >> 1);
                            o[2 * g8] = v0;
                            o[2 * (g8 + 8)] = v1;
                        }
                    }
                }
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
            if (GLU) {
                // pairs (gate tile 2 jp, up tile 2 jp + 1) of the tile-group
                const int npo = (nt >> 1) * CS * 32;
                for (int o = threadIdx.x; o < npo; o += kConsumers * 32) {
                    const int jp = o / (CS * 32), rem = o % (CS * 32);
                    float vg = 0.f, vu = 0.f;
#pragma unroll
                    for (int ww = 0; ww < kGroupWarps; ww++) {
                        vg += rb[ww * TB * CS * 32 + (2 * jp) * CS * 32 + rem];
                        vu += rb[ww * TB * CS * 32 + (2 * jp + 1) * CS * 32 + rem];
                    }
                    const int tok = 2 * (rem >> 5) + (rem & 1), row = (rem & 31) >> 1;
                    const int64_t n = (int64_t)((tb >> 1) + jp) * 16 + row;
                    if (ok && tok < M && n < N)
                        store_y<float>(y, yt, (int64_t)tok * N + n, vg / (1.f + expf(-vg)) * vu);
                }
                continue;
            }
            const int nout = nt * CS * 32;
            for (int o = threadIdx.x; o < nout; o += kConsumers * 32) {
                float v = 0.f;
#pragma unroll
                for (int ww = 0; ww < kGroupWarps; ww++)
                    v += rb[ww * TB * CS * 32 + o];
                const int j = o / (CS * 32), rem = o % (CS * 32);
                const int tok = 2 * (rem >> 5) + (rem & 1), row = (rem & 31) >> 1;
                const int64_t n = (int64_t)(tb + j) * 16 + row;
                if (TOPK) {
                    if (tok < M)
                        lgp[tok * tp.lg_rows + (tb - t0 + j) * 16 + row] = v;
                } else if (ok && tok < M && n < N) {
                    store_y<float>(y, yt, (int64_t)tok * N + n, v);
                }
            }
        }
        if (TOPK)
            topk_tail<kConsumers * 32>(tp, lgp, reinterpret_cast<topk::Smem *>(smem + L.tks),
                                       reinterpret_cast<unsigned long long *>(smem + L.tko), M, N, t0, t1, ok,
                                       reinterpret_cast<unsigned long long *>(ring), S * L.stage_bytes);
    }
    if (threadIdx.x == 0) {
        // the bulk copy this thread issued must have landed before the CTA exits
        volatile int no_abort = 0;
        ptx::mbar_wait_bounded(&bars->frag, 0, &no_abort, err, kDevErrTimeout, kWaitLimitNs);
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_rows()
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

int sm_count_rows()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

struct RPlan {
    int CS, WG, TB, S, grid, T, smem;
    int lg_rows;                                  // top-k: rows of the per-CTA logits buffer (0: plain GEMV)
    bool lg_glob;                                 // top-k: logits in the workspace (too large for shared memory)
    size_t frag_bytes, colf_bytes, cfix_bytes;
    size_t cand_bytes, counter_bytes;             // top-k: candidates [grid][M][k] u64, the ticket counter
    size_t lg_bytes;                              // top-k with lg_glob: [grid][M][lg_rows] f32
};

template <int FMT, int CS>
int rows_total(int G, int TB, int S, int lg) { return rows_layout<FMT, CS>(G, TB, S, lg < 0 ? 0 : lg, lg != 0).total; }

// lg: the top-k logits kept in shared memory (> 0), top-k with them in the workspace (< 0), or a
// plain GEMV (0)
int rows_total_rt(int fmt, int CS, int G, int TB, int S, int lg)
{
    if (fmt == BQ_TERNARY_B3_G128)
        return CS == 1 ? rows_total<BQ_TERNARY_B3_G128, 1>(G, TB, S, lg) : CS == 2 ? rows_total<BQ_TERNARY_B3_G128, 2>(G, TB, S, lg)
             : CS == 3 ? rows_total<BQ_TERNARY_B3_G128, 3>(G, TB, S, lg) : rows_total<BQ_TERNARY_B3_G128, 4>(G, TB, S, lg);
    if (fmt == BQ_BINARY_G128)
        return CS == 1 ? rows_total<BQ_BINARY_G128, 1>(G, TB, S, lg) : CS == 2 ? rows_total<BQ_BINARY_G128, 2>(G, TB, S, lg)
             : CS == 3 ? rows_total<BQ_BINARY_G128, 3>(G, TB, S, lg) : rows_total<BQ_BINARY_G128, 4>(G, TB, S, lg);
    return CS == 1 ? rows_total<BQ_TERNARY_G128, 1>(G, TB, S, lg) : CS == 2 ? rows_total<BQ_TERNARY_G128, 2>(G, TB, S, lg)
         : CS == 3 ? rows_total<BQ_TERNARY_G128, 3>(G, TB, S, lg) : rows_total<BQ_TERNARY_G128, 4>(G, TB, S, lg);
}

// Tiles per tile-group: as many as a CTA owns, up to 4 per warp group; two warp groups (16
// consumer warps) at one column set when a CTA owns at least 8 tiles, where the stream is long
// and more warps hide more latency (on the 248320-row LM head 8 warps measured 58% slower than
// 16; 24 warps, at 80 registers a thread, 5% slower). Stages: as many as fit, preferring (with one warp group) a
// footprint that lets two CTAs share an SM, so that the next call's CTA can become resident and
// prefetch while this one runs; 0 stages if even three do not fit.
// Top-k (topk_k > 0) adds the CTA's logits [M][per * 16] and the selection scratch to shared
// memory, and the candidates and the ticket counter to the workspace.
static RPlan rows_plan_lg(int M, int fmt, int64_t N, int64_t K, int topk_k, bool lg_glob, bool glu = false);

// Top-k keeps the CTA's logits in shared memory when that costs no pipeline stage, else in the
// workspace, where they stay in L2 (at most 148 x 8 x 1680 x 4 bytes at the LM head); the
// selection then reads them from L2.
RPlan rows_plan(int M, int fmt, int64_t N, int64_t K, int topk_k)
{
    if (topk_k <= 0)
        return rows_plan_lg(M, fmt, N, K, 0, false);
    const RPlan on_chip = rows_plan_lg(M, fmt, N, K, topk_k, false);
    const RPlan in_ws = rows_plan_lg(M, fmt, N, K, topk_k, true);
    return on_chip.S >= 3 && on_chip.S >= in_ws.S ? on_chip : in_ws;
}

// glu: N gate rows, 2 ceil(N / 16) logical tiles in gate/up pairs; CTAs and tile-groups take
// whole pairs, so per and TB are even.
static RPlan rows_plan_lg(int M, int fmt, int64_t N, int64_t K, int topk_k, bool lg_glob, bool glu)
{
    RPlan p{};
    p.lg_glob = lg_glob;
    p.CS = (M * kColsPerTok + 7) / 8;
    const int G = (int)(K / 128);
    const int units = (int)((N + 15) / 16);               // tiles, or gate/up pairs
    p.T = glu ? 2 * units : units;
    const int sms = sm_count_rows();
    p.grid = units < sms ? units : sms;
    const int per_units = (units + p.grid - 1) / p.grid;
    const int per = glu ? 2 * per_units : per_units;
    p.lg_rows = topk_k > 0 ? per * 16 : 0;
    const int lg = topk_k > 0 ? (lg_glob ? -1 : M * p.lg_rows) : 0;
    p.WG = p.CS == 1 && per >= 2 * kWarpTiles ? 2 : 1;
    // as many tiles per tile-group as a warp group can take, the CTA's tiles spread evenly over
    // its tile-groups (9 tiles: 5 + 4, not 8 + 1), and fewer if three stages do not fit
    for (int tbmax = kWarpTiles * p.WG; tbmax >= (glu ? 2 : 1); tbmax -= glu ? 2 : 1) {
        if (glu) {
            const int ntg = (per_units + tbmax / 2 - 1) / (tbmax / 2);
            p.TB = 2 * ((per_units + ntg - 1) / ntg);
        } else {
            const int ntg = (per + tbmax - 1) / tbmax;
            p.TB = (per + ntg - 1) / ntg;
        }
        p.S = 0;
        if (p.WG == 1)
            for (int s = kMaxStages; s >= 3; s--)
                if (rows_total_rt(fmt, p.CS, G, p.TB, s, lg) <= kSmemPair) {
                    p.S = s;
                    break;
                }
        if (p.S < 4) {
            for (int s = kMaxStages; s >= 3; s--)
                if (rows_total_rt(fmt, p.CS, G, p.TB, s, lg) <= kSmemLimit) {
                    p.S = s;
                    break;
                }
        }
        if (p.S >= 3)
            break;
    }
    p.smem = p.S ? rows_total_rt(fmt, p.CS, G, p.TB, p.S, lg) : 0;
    auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
    p.frag_bytes = al((size_t)p.CS * G * 1024);
    p.colf_bytes = al((size_t)2 * p.CS * G * 4);
    p.cfix_bytes = al((size_t)p.CS * G * 32);
    p.cand_bytes = topk_k > 0 ? al((size_t)p.grid * M * (topk_k + 1) * 8) : 0;
    p.counter_bytes = topk_k > 0 ? 256 : 0;
    p.lg_bytes = topk_k > 0 && lg_glob ? al((size_t)p.grid * M * p.lg_rows * 4) : 0;
    return p;
}

// The up matrix of a GLU launch (same format, shape and layout as a.words / a.scales).
struct GluUp {
    const uint32_t *words;
    const __half *scales;
};

template <int FMT>
CUresult encode_weight_maps(EncodeTiledFn enc, const uint32_t *words, const __half *scales, int64_t N, int64_t K,
                            CUtensorMap *mw, CUtensorMap *ms)
{
    const cuuint64_t G = (cuuint64_t)(K / 128);
    cuuint32_t est[2] = {1, 1};
    CUresult r;
    if (FMT == BQ_TERNARY_B3_G128) {
        // bytes [N][26 G]; a box is one 208-byte block (8 groups) of 16 rows, unswizzled: at a
        // 208-byte pitch the 8 rows a warp reads fall in distinct banks
        const cuuint64_t rb = (cuuint64_t)b3::kGroupBytes * G;
        cuuint64_t wdims[2] = {rb, (cuuint64_t)N};
        cuuint64_t wstr[1] = {rb};
        cuuint32_t wbox[2] = {(cuuint32_t)b3::kBlockBytes, 16};
        r = enc(mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint32_t *>(words), wdims, wstr, wbox, est,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        const cuuint64_t wpr = (cuuint64_t)(FMT == BQ_BINARY_G128 ? K / 32 : K / 16);
        cuuint64_t wdims[2] = {wpr, (cuuint64_t)N};
        cuuint64_t wstr[1] = {wpr * 4};
        cuuint32_t wbox[2] = {32, 16};                   // 128 bytes x 16 rows
        r = enc(mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(words), wdims, wstr, wbox, est,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS)
        return r;
    cuuint64_t sdims[2] = {G, (cuuint64_t)N};
    cuuint64_t sstr[1] = {G * 2};
    cuuint32_t sbox[2] = {8, 16};                        // the 8 scales of a 1024-k slice x 16 rows
    return enc(ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<__half *>(scales), sdims, sstr, sbox, est,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

template <int FMT, int CS, int WG, typename XT>
cudaError_t launch_rows_t(const GemvArgs &a, const RPlan &pl, cudaStream_t s, const TopkParams *tk,
                          const GluUp *glu)
{
    EncodeTiledFn enc = encode_fn_rows();
    if (!enc)
        return cudaErrorNotSupported;
    const cuuint64_t G = (cuuint64_t)(a.K / 128);
    CUtensorMap mw, ms, mw2, ms2;
    if (encode_weight_maps<FMT>(enc, a.words, a.scales, a.N, a.K, &mw, &ms) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    if (glu) {
        if (encode_weight_maps<FMT>(enc, glu->words, glu->scales, a.N, a.K, &mw2, &ms2) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    } else {
        mw2 = mw;
        ms2 = ms;
    }
    auto kern = tk ? gemv_rows_kernel<FMT, CS, WG, kModeTopk>
              : glu ? gemv_rows_kernel<FMT, CS, WG, kModeGlu> : gemv_rows_kernel<FMT, CS, WG, kModePlain>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess)
        return e;
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    uint32_t *frag = reinterpret_cast<uint32_t *>(ws);
    float *colf = reinterpret_cast<float *>(ws + pl.frag_bytes);
    int *cfix = reinterpret_cast<int *>(ws + pl.frag_bytes + pl.colf_bytes);
    TopkParams tp{};
    unsigned int *counter = nullptr;
    if (tk) {
        tp = *tk;
        uint8_t *tw = ws + pl.frag_bytes + pl.colf_bytes + pl.cfix_bytes;
        tp.cand = reinterpret_cast<unsigned long long *>(tw);
        tp.counter = counter = reinterpret_cast<unsigned int *>(tw + pl.cand_bytes);
        tp.lg_rows = pl.lg_rows;
        tp.lg_glob = pl.lg_glob ? reinterpret_cast<float *>(tw + pl.cand_bytes + pl.counter_bytes) : nullptr;
    }
    // programmatic dependent launches: each kernel may start before its predecessor in the
    // stream has finished, and waits for it (griddepcontrol.wait) before reading x or the
    // fragments, or writing anything
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t pcfg = {};
    const int items = (int)G * a.M;
    pcfg.gridDim = dim3((unsigned)((items * 32 + 255) / 256));
    pcfg.blockDim = dim3(256);
    pcfg.stream = s;
    pcfg.attrs = attr;
    pcfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&pcfg, gemv_rows_prep_kernel<FMT, CS, XT>, static_cast<const XT *>(a.x), a.M, a.K, frag,
                           colf, cfix, counter);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.grid);
    cfg.blockDim = dim3((WG * kGroupWarps + 1) * 32);
    cfg.dynamicSmemBytes = (size_t)pl.smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mw, ms, mw2, ms2, a.M, a.N, a.K, a.y, a.yt, pl.T, pl.TB, pl.S,
                              (const uint32_t *)frag, (const float *)colf, (const int *)cfix, 1u, a.dev_status,
                              a.wait_ns, tp);
}

template <int FMT, typename XT>
cudaError_t launch_rows_cs(const GemvArgs &a, const RPlan &pl, cudaStream_t s, const TopkParams *tk,
                           const GluUp *glu)
{
    switch (pl.CS) {
    case 1:
        return pl.WG == 2 ? launch_rows_t<FMT, 1, 2, XT>(a, pl, s, tk, glu) : launch_rows_t<FMT, 1, 1, XT>(a, pl, s, tk, glu);
    case 2: return launch_rows_t<FMT, 2, 1, XT>(a, pl, s, tk, glu);
    case 3: return launch_rows_t<FMT, 3, 1, XT>(a, pl, s, tk, glu);
    default: return launch_rows_t<FMT, 4, 1, XT>(a, pl, s, tk, glu);
    }
}

}  // namespace

// K a multiple of 1024 (whole 8-scale slices) and the digit fragments of all of K in shared
// memory next to at least three stages.
bool gemv_rows_supported(int M, int fmt, int64_t N, int64_t K, int topk_k)
{
    if (M < 1 || M > 8 || K % 1024 != 0 || N < 1)
        return false;
    return rows_plan(M, fmt, N, K, topk_k).S >= 3;
}

size_t gemv_rows_workspace_bytes(int M, int fmt, int64_t N, int64_t K, int topk_k)
{
    const RPlan p = rows_plan(M, fmt, N, K, topk_k);
    return p.frag_bytes + p.colf_bytes + p.cfix_bytes + p.cand_bytes + p.counter_bytes + p.lg_bytes;
}

template <int FMT>
static cudaError_t launch_rows_x(const GemvArgs &a, const RPlan &pl, cudaStream_t s, const TopkParams *tk,
                                 const GluUp *glu)
{
    if (a.xt == BQ_F16)
        return launch_rows_cs<FMT, __half>(a, pl, s, tk, glu);
    if (a.xt == BQ_BF16)
        return launch_rows_cs<FMT, __nv_bfloat16>(a, pl, s, tk, glu);
    return launch_rows_cs<FMT, float>(a, pl, s, tk, glu);
}

// Plain GEMV (tk, glu null), the top-k GEMV, or the gate/up projection with SwiGLU.
static cudaError_t launch_rows_any(const GemvArgs &a, cudaStream_t s, const TopkParams *tk, const GluUp *glu = nullptr)
{
    const RPlan pl = glu ? rows_plan_lg(a.M, a.fmt, a.N, a.K, 0, false, true) : rows_plan(a.M, a.fmt, a.N, a.K, tk ? tk->k : 0);
    if (a.fmt == BQ_BINARY_G128)
        return launch_rows_x<BQ_BINARY_G128>(a, pl, s, tk, glu);
    if (a.fmt == BQ_TERNARY_B3_G128)
        return launch_rows_x<BQ_TERNARY_B3_G128>(a, pl, s, tk, glu);
    return launch_rows_x<BQ_TERNARY_G128>(a, pl, s, tk, glu);
}

bool gemv_glu_supported(int M, int fmt, int64_t N, int64_t K)
{
    if (M < 1 || M > 8 || K % 1024 != 0 || N < 1)
        return false;
    return rows_plan_lg(M, fmt, N, K, 0, false, true).S >= 3;
}

size_t gemv_glu_workspace_bytes(int M, int fmt, int64_t N, int64_t K)
{
    const RPlan p = rows_plan_lg(M, fmt, N, K, 0, false, true);
    return p.frag_bytes + p.colf_bytes + p.cfix_bytes;
}

cudaError_t launch_gemv_glu(const GemvArgs &a, const uint32_t *up_words, const __half *up_scales, cudaStream_t s,
                            unsigned *launches)
{
    *launches = 2;                                        // digit prep + the gate/up GEMV with SwiGLU
    const GluUp up{up_words, up_scales};
    return launch_rows_any(a, s, nullptr, &up);
}

cudaError_t launch_gemv_rows(const GemvArgs &a, cudaStream_t s, unsigned *launches)
{
    *launches = 2;                                        // digit prep + the GEMV
    return launch_rows_any(a, s, nullptr);
}

cudaError_t launch_gemv_topk(const GemvArgs &a, const TopkArgs &t, cudaStream_t s, unsigned *launches)
{
    *launches = 2;                                        // digit prep + the GEMV with its selection
    TopkParams tp{};
    tp.k = t.k;
    tp.vals = t.vals;
    tp.idx = t.idx;
    tp.u = t.u;
    tp.temp = t.temperature;
    tp.top_p = t.top_p;
    tp.tokens = t.tokens;
    return launch_rows_any(a, s, &tp);
}

// ---------------------------------------------------------------------------------------
// fixed scratch of bq_gemv_noalloc
// ---------------------------------------------------------------------------------------
// The scratch this GEMV needs is the digit fragments, factors and accumulator inputs of x, which
// by construction fit in one CTA's shared memory (227 KB), plus their 256-byte alignment. This
// array holds the largest such set. Nothing in it needs an initial value: every call's prep
// kernel writes what the GEMV then reads.
constexpr size_t kStaticScratchBytes = 256 * 1024;
static __device__ __align__(256) unsigned char g_gemv_scratch[kStaticScratchBytes];

cudaError_t gemv_static_scratch(void **ptr, size_t *bytes)
{
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static void *addr[kMaxDev] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        // first use on this device (the device is current): resolve the array's address
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_gemv_scratch);
        if (e != cudaSuccess)
            return e;
        addr[dev] = p;
    }
    *ptr = addr[dev];
    *bytes = sizeof(g_gemv_scratch);
    return cudaSuccess;
}

}  // namespace bq
