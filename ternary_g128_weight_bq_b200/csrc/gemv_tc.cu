// gemv_tc.cu -- decode GEMV (M <= 8) on packed binary-g128 / ternary-g128 weights that streams
// the packed words at HBM speed and sums on the integer tensor cores.
//
// Model card "prism-ml/Bonsai-27B-mlx-1bit", sections "Weight representation: Binary g128" and
// "CUDA (NVIDIA GPUs)": y[m][n] = sum_g s[n][g] * sum_{k in g} v[n][k] x[m][k], v = +-1
// (binary) or {-1, 0, +1} (ternary: "Ternary Bonsai 27B vs ..." article, wmrh.cn); the packed
// weights are unpacked inside the product and each group scale is applied once per group.
// Batch-1 decode (tg128) is the memory-bound phase of section "Cross-platform throughput".
//
// Why this shape. At B200's HBM rate one SM receives ~174 binary weights per clock. A
// select-and-add per weight on the CUDA cores costs more issue slots than that, so the sign
// bits go to mma.sync m16n8k32 s8 (measured ~177 weights per SM clock with fresh operands),
// which does the additions exactly in int32: the "add" of select-and-add runs on the tensor
// pipe. A binary register of four weights is one AND of the word (or of the word shifted by 3
// or 6 bits) with a byte mask: bit b of a byte becomes b * 2^p, p in {5, 6, 7}; two shifts and
// eight ANDs per 32 weights. Ternary codes become {-64, 0, +64} with one PRMT per four codes.
//
// x as integers. Per (token, group of 128), x is written as X = round(x * 2^(21-e)) with
// e = floor(log2 max|x|) over the group, |X| < 2^22, split into balanced digits: four of base
// 64 for binary (|d| <= 32; the B byte is d * 2^(7-p), so each product is 128 b d, and the
// accumulator starts at -64 sum(d) over the group, which turns sum(b d) into the sum of
// (2b - 1) d / 2), three of base 256 and a zero column for ternary. Every digit is one MMA
// column; a token owns four. The rounding error is at most 2^-22 max|x| per element,
// 2^-15 max|x| s per group: below 1/60 of that group's share of the 2e-3 sum|x s| tolerance.
// The int32 column sums are exact (each also starts at the bits of 1.5 * 2^23, so one fp32
// subtraction turns it into a float without rounding); the group scale times 2^(e-27) is
// applied once per group in fp32, and the digit weight once per block.
//
// Two kernels per call, both with programmatic dependent launch:
//   * a prep kernel turns x into the MMA B fragments (digits), the per-(token, group) factors
//     and accumulator inputs once, one warp per (group, token slot), and zeroes the split-block
//     counters; every CTA of the GEMV then bulk-copies the fragments of the k-chunks it touches
//     into shared memory (building them in each CTA cost up to 25 us at M = 8, all of it after
//     the previous kernel had finished), while its producer already streams the first weight
//     tiles;
//   * units = (block of ROWS rows, one stage of k); CTA i owns units [i U / P, (i+1) U / P)
//     (stream-K), so every shape is balanced to one unit;
//   * the producer lane TMA-loads, per unit, a ROWS x 128 bytes tile of packed words (1024
//     binary / 512 ternary weights per row; 128B swizzle; 128-byte rows stream measurably
//     faster than 64-byte ones) into a ring of stages; one consumer warp per 16-row tile
//     expands the stage's groups two or four at a time (independent MMA chains); the group
//     scales come straight from global memory, each stage's loaded one stage early;
//   * a block owned by one CTA is written directly; a block split between CTAs leaves partial
//     sums in the workspace (two block slots per CTA: its first and its last block), and the
//     last warp to finish its 16 rows (one atomic on a counter the prep kernel zeroed) adds
//     them in a fixed order.
#include <cuda.h>

#include <mutex>

#include "bq_internal.cuh"
#include "sm100_ptx.cuh"

namespace bq {
namespace {

// A block is ROWS weight rows: one consumer warp per 16-row tile plus one producer warp.
// 192 rows (12 consumer warps, registers capped at 128 by the 13-warp block) at one column set,
// where more warps hide more latency; 128 rows (8 consumer warps, up to 168 registers) where
// the wider accumulators of two to four column sets need the registers.
template <int ROWS> struct Geo {
    static constexpr int kRows = ROWS;
    static constexpr int kTiles = ROWS / 16;
    static constexpr int kConsumers = kTiles;
    static constexpr int kThreads = (kConsumers + 1) * 32;
};
constexpr int rows_for(int fmt, int CS) { return fmt == BQ_BINARY_G128 && CS == 1 ? 192 : 128; }
constexpr int kMaxTiles = 12;
constexpr int kColsPerTok = 4;       // MMA columns per token (one per digit of x; see Digits)
constexpr int kMagic = 0x4B400000;   // bits of 1.5 * 2^23: int n in |n| < 2^22 -> float(bits + n) = 1.5*2^23 + n
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 227 * 1024;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

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

// One stage = 128 rows x 128 bytes of packed words (one 128-byte-swizzled TMA box):
// 1024 k (8 groups) of binary weights or 512 k (4 groups) of ternary codes.
template <int FMT, int ROWS> struct StageCfg {
    static constexpr int kGroups = FMT == BQ_BINARY_G128 ? 8 : 4;
    static constexpr int kBytes = ROWS * 128;
};

// How x and the weights enter the MMA.
//   kMask (binary, one column set, where the expansion is most of the work): four balanced
//     base-64 digits per token (|d| <= 32); the sign bits enter as b * 2^p with b in {0, 1}
//     (one AND per four weights, p = 5, 6 or 7 by register) and the B byte is d * 2^(7-p)
//     (negated for p = 7, where b * 2^7 is the s8 value -128), so every product is 128 b d; the
//     -64 sum(d) that turns b into 2b - 1 is the MMA's accumulator input, a per-(group, column)
//     value.
//   otherwise (binary at two to four column sets, where the tensor pipe is the limit and a
//     per-group accumulator input would cost a load per column set; ternary): three balanced
//     base-256 digits and a zero column; sign bits enter as +-64 (one shift and one LOP3 per
//     four weights), ternary codes as {-64, 0, +64} (one PRMT per four codes); the accumulator
//     input is a constant.
template <int FMT, int CS> struct Scheme {
    static constexpr bool kMask = FMT == BQ_BINARY_G128 && CS == 1;
    static constexpr int kCount = kMask ? 4 : 3;
    static constexpr int kBits = kMask ? 6 : 8;
    static constexpr int kRows = rows_for(FMT, CS);
};

// Binary: bit position p that bit (8b + rho) of a word lands on in A register rho, and the
// matching B multiplier 2^(7-p) (-1 for p = 7).
__host__ __device__ constexpr int bin_p(int rho) { return rho == 2 || rho == 5 ? 5 : (rho == 0 || rho == 3 || rho == 6 ? 6 : 7); }
__host__ __device__ constexpr int bin_bmul(int rho) { return bin_p(rho) == 5 ? 4 : (bin_p(rho) == 6 ? 2 : -1); }

struct Layout {
    int frag_off, colf_off, cfix_off, stage_off, red_off, bar_off, total, stages;
};

// Shared-memory layout for a call (host and device compute the same thing).
template <int FMT, int CS, int ROWS>
__host__ __device__ inline Layout make_layout(int G, int stages)
{
    Layout L;
    L.frag_off = 0;
    L.colf_off = CS * G * 1024;
    L.cfix_off = L.colf_off + 2 * CS * G * 4;                           // one factor per token slot
    L.stage_off = (L.cfix_off + CS * G * 32 + 1023) / 1024 * 1024;      // accumulator inputs [cs][q][8]
    L.red_off = L.stage_off + stages * StageCfg<FMT, ROWS>::kBytes;
    L.bar_off = L.red_off + Geo<ROWS>::kTiles * 16 * CS * 8 * 4;
    L.total = L.bar_off + 256 + 1024;                // barriers + alignment slack
    L.stages = stages;
    return L;
}

struct Bars {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t frag;                    // the digit fragments and factors have landed
    int abort;
};

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

// 8 A registers (s8 +-64) of one binary word: register i holds, in byte b, bit 8b + i
// (1 -> +64 = 0x40, 0 -> -64 = 0xC0). The shift is a multiply by mul[i] = 2^(7-i) held in a
// register, so it issues on the FMA pipe; the LOP3 issues on the ALU pipe.
// mul = {2^7, .., 2^1, 0x80808080, 0x40404040}: the masks live in registers (they come from a
// kernel argument), so each byte select is a single three-register LOP3.
__device__ __forceinline__ void expand_binary_pm64(uint32_t w, const uint32_t (&mul)[9], uint32_t *a)
{
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const uint32_t sh = i < 7 ? w * mul[i] : w;  // bit 8b+i -> 8b+7 (mul[i] = 2^(7-i), a register)
        uint32_t r;
        asm("lop3.b32 %0, %1, %2, %3, 0xAE;" : "=r"(r) : "r"(sh), "r"(mul[7]), "r"(mul[8]));
        a[i] = r;                                    // (~sh & 0x80808080) | 0x40404040
    }
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
    uint32_t a0[8], a1[8];
    if (FMT == BQ_BINARY_G128 && MASK) {
        expand_binary_mask(*reinterpret_cast<const uint32_t *>(p0), mul, a0);
        expand_binary_mask(*reinterpret_cast<const uint32_t *>(p1), mul, a1);
    } else if (FMT == BQ_BINARY_G128) {
        expand_binary_pm64(*reinterpret_cast<const uint32_t *>(p0), mul, a0);
        expand_binary_pm64(*reinterpret_cast<const uint32_t *>(p1), mul, a1);
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

// Digit fragments of token slot m (MMA columns 4m .. 4m+3) in group q, the token's factor
// 2^(e-27) (the weight 2^(kBits d) of digit d is applied per block) and the accumulator inputs
// of its columns (the bits of 1.5 * 2^23, minus 64 sum(d) over the group for binary), written
// with the shared-memory layouts [cs][q][half][lane][4] u32, [slot][G] f32 and [cs][q][8] s32.
// One warp; lane (t, rho) builds register rho of quad-thread t. Slots m >= M (the padding of
// the last column set) get zeros, so a quad-thread's two accumulator columns always belong to
// one token.
template <int FMT, int CS, typename XT>
__device__ __forceinline__ void build_token(const XT *__restrict__ x, int M, int64_t K, int G, int q, int m,
                                            int lane, uint32_t *__restrict__ frag, float *__restrict__ colf,
                                            int *__restrict__ cfix)
{
    using D = Scheme<FMT, CS>;
    const int t = lane >> 3, rho = lane & 7;
    uint32_t dw[4] = {0u, 0u, 0u, 0u};
    int csum[4] = {0, 0, 0, 0};
    float fac = 0.f;
    if (m < M) {
        float v[4];
#pragma unroll
        for (int b = 0; b < 4; b++)
            v[b] = load_x(x + (int64_t)m * K + 128 * q + k_local<FMT>(t, rho, b));
        float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
        for (int o = 16; o; o >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        int e = 0;
        if (amax > 0.f) {
            frexpf(amax, &e);                        // amax = f 2^e, f in [0.5, 1)
            e -= 1;                                  // amax in [2^e, 2^(e+1))
        }
        const int bmul = D::kMask ? bin_bmul(rho) : 1;
#pragma unroll
        for (int b = 0; b < 4; b++) {
            int X = amax > 0.f ? __float2int_rn(ldexpf(v[b], 21 - e)) : 0;   // |X| < 2^22
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
#pragma unroll
                for (int o = 16; o; o >>= 1)
                    csum[d] += __shfl_xor_sync(0xffffffffu, csum[d], o);
        }
        fac = amax > 0.f ? ldexpf(1.f, e - 27) : 0.f;                       // 2^(e-21) / 64
    }
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

// x -> digit fragments and factors of every (group, token slot), once per call, into the
// workspace; block 0 also zeroes the split-block counters. One warp per (group, slot).
constexpr int kPrepThreads = 256;

template <int FMT, int CS, typename XT>
__global__ void __launch_bounds__(kPrepThreads)
gemv_prep_kernel(const XT *__restrict__ x, int M, int64_t K, uint32_t *__restrict__ frag,
                 float *__restrict__ colf, int *__restrict__ cfix, unsigned int *__restrict__ counters,
                 int n_counters)
{
    // the GEMV that reads these fragments may start its weight stream now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // x may be the output of the previous kernel, and the previous GEMV may still be reading
    // the workspace: wait for it to finish before writing anything
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int G = (int)(K / 128);
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < n_counters; i += kPrepThreads)
            counters[i] = 0u;
    const int item = (int)((blockIdx.x * kPrepThreads + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (item < G * 2 * CS)
        build_token<FMT, CS, XT>(x, M, K, G, item / (2 * CS), item % (2 * CS), lane, frag, colf, cfix);
}

template <int FMT, int CS, int ROWS>
__global__ void __launch_bounds__(Geo<ROWS>::kThreads, 1)
gemv_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const uint16_t *__restrict__ scales,
               int M, int64_t N, int64_t K, void *__restrict__ y, int yt,
               float *__restrict__ part, unsigned int *__restrict__ counters,
               const uint32_t *__restrict__ frag_g, const float *__restrict__ colf_g,
               const int *__restrict__ cfix_g, int64_t U, int C,
               int stages, uint32_t one, unsigned int *dev_status)
{
    using SC = StageCfg<FMT, ROWS>;
    using SCH = Scheme<FMT, CS>;
    constexpr int kRows = ROWS, kTiles = Geo<ROWS>::kTiles, kConsumers = Geo<ROWS>::kConsumers;
    const int G = (int)(K / 128);
    const Layout L = make_layout<FMT, CS, ROWS>(G, stages);
    const int S = stages;
    extern __shared__ uint8_t smem_raw[];
    // align by an offset on the shared array itself, so every access stays a shared-memory one
    uint8_t *smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint32_t *frag_s = reinterpret_cast<uint32_t *>(smem + L.frag_off);
    float *colf_s = reinterpret_cast<float *>(smem + L.colf_off);
    int *cfix_s = reinterpret_cast<int *>(smem + L.cfix_off);
    float *red = reinterpret_cast<float *>(smem + L.red_off);
    Bars *bars = reinterpret_cast<Bars *>(smem + L.bar_off);
    volatile int *abort = &bars->abort;
    unsigned int *err = dev_status + kSlotErrBits;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t Pn = gridDim.x;
    const int64_t u0 = (int64_t)blockIdx.x * U / Pn, u1 = ((int64_t)blockIdx.x + 1) * U / Pn;

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
    // the next kernel in the stream may start its own prologue now; it still waits for this
    // grid to finish before it reads anything this grid writes
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == kConsumers) {
        // ------------------------------------------------------------------- producer
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tmap_w);
            int64_t it = 0;
            int s = 0;
            uint32_t ph = 0;
            int64_t rb = u0 / C;
            int c = (int)(u0 % C);
            for (int64_t u = u0; u < u1; u++, it++) {
                // a free slot: the producer sleeps in the wait, leaving the issue slots to the consumers
                if (!ptx::mbar_wait_bounded_sleep(&bars->empty[s], ph ^ 1, abort, err, kDevErrTimeout, kWaitLimitNs))
                    break;
                uint8_t *st = smem + L.stage_off + s * SC::kBytes;
                ptx::mbar_arrive_expect_tx(&bars->full[s], SC::kBytes);
                ptx::tma_load_2d(st, &tmap_w, &bars->full[s], c * 32, (int32_t)(rb * kRows));
                if (++s == S) {
                    s = 0;
                    ph ^= 1;
                }
                if (++c == C) {
                    c = 0;
                    rb++;
                }
            }
            // no copy may still be in flight when the CTA exits
            for (int64_t k = it > S ? it - S : 0; k < it; k++) {
                volatile int no_abort = 0;
                ptx::mbar_wait_bounded(&bars->full[k % S], (uint32_t)((k / S) & 1), &no_abort, err,
                                       kDevErrTimeout, kWaitLimitNs);
            }
        }
    } else {
        // ------------------------------------------------------------------- consumers
        // the fragments are written by the prep kernel launched just before this one
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (threadIdx.x == 0) {
            // bulk-copy the digit fragments of the k-chunks this CTA touches (one range, two
            // when its units wrap into the next row block, all of them if it owns >= C units)
            // and all the factors
            int ra0 = 0, ra1 = C, rb0 = 0, rb1 = 0;
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
            constexpr uint32_t kChunkBytes = SC::kGroups * 1024;
            const uint32_t colf_bytes = (uint32_t)(2 * CS * G * 4), cfix_bytes = (uint32_t)(CS * G * 32);
            ptx::mbar_arrive_expect_tx(&bars->frag, (uint32_t)CS * (uint32_t)(ra1 - ra0 + rb1 - rb0) * kChunkBytes +
                                                        colf_bytes + cfix_bytes);
#pragma unroll
            for (int cs = 0; cs < CS; cs++) {
                const size_t o = (size_t)cs * G * 256;
                ptx::bulk_load(frag_s + o + ra0 * SC::kGroups * 256, frag_g + o + ra0 * SC::kGroups * 256,
                               (uint32_t)(ra1 - ra0) * kChunkBytes, &bars->frag);
                if (rb1 > rb0)
                    ptx::bulk_load(frag_s + o, frag_g + o, (uint32_t)(rb1 - rb0) * kChunkBytes, &bars->frag);
            }
            ptx::bulk_load(colf_s, colf_g, colf_bytes, &bars->frag);
            ptx::bulk_load(cfix_s, cfix_g, cfix_bytes, &bars->frag);
        }

        const int tile = warp;                          // this warp's 16-row tile; it takes every group
        const int g8 = lane >> 2, t = lane & 3;
        const int r0 = tile * 16 + g8, r1 = r0 + 8;          // rows of this thread in the block
        // shift multipliers and byte masks of the binary expansion: runtime values, kept in registers
        uint32_t mul[9];
        if (SCH::kMask) {
            mul[0] = one * 8u;
            mul[1] = one * 64u;
            mul[2] = one * 0x20202020u;
            mul[3] = one * 0x40404040u;
            mul[4] = one * 0x80808080u;
            mul[5] = mul[6] = mul[7] = mul[8] = 0u;
        } else {
#pragma unroll
            for (int i = 0; i < 7; i++)
                mul[i] = one << (7 - i);
            mul[7] = one * 0x80808080u;
            mul[8] = one * 0x40404040u;
        }
        const int m0 = (int)(one - 1u) + kMagic;        // constant accumulator input (not kMask)
        const int magic[4] = {m0, m0, m0, m0};
        // the stage's groups, GP at a time
        constexpr int GH = SC::kGroups;
        // byte offsets of this thread's packed word(s) of each of those groups in rows r0 / r1
        // (128-byte rows, 128B swizzle: 16-byte chunk j of row r sits at j ^ (r & 7))
        int woff[GH][2];
#pragma unroll
        for (int h = 0; h < GH; h++) {
            const int q = h;
            const int j = FMT == BQ_BINARY_G128 ? q : 2 * q + (t >> 1);          // 16-byte chunk
            const int within = FMT == BQ_BINARY_G128 ? 4 * t : 8 * (t & 1);
            woff[h][0] = r0 * 128 + ((j ^ (r0 & 7)) << 4) + within;
            woff[h][1] = r1 * 128 + ((j ^ (r1 & 7)) << 4) + within;
        }
        // this thread's GH scales of rows r0 / r1, loaded one stage before they are needed:
        // row pointers are set once per block (rows past N read row 0 and are zeroed)
        struct ScaleRows {
            const uint16_t *p0, *p1;
            bool v0, v1;
        };
        auto scale_rows = [&](int64_t rb_) {
            const int64_t n0 = rb_ * kRows + r0, n1 = n0 + 8;
            ScaleRows sr;
            sr.v0 = n0 < N;
            sr.v1 = n1 < N;
            sr.p0 = scales + (sr.v0 ? n0 : 0) * G;
            sr.p1 = scales + (sr.v1 ? n1 : 0) * G;
            return sr;
        };
        auto load_scales = [&](const ScaleRows &sr, int c_, uint32_t (&o0)[GH / 2], uint32_t (&o1)[GH / 2]) {
            const uint16_t *p0 = sr.p0 + c_ * SC::kGroups, *p1 = sr.p1 + c_ * SC::kGroups;
            if (GH == 8) {
                const uint4 a = sr.v0 ? __ldg(reinterpret_cast<const uint4 *>(p0)) : make_uint4(0, 0, 0, 0);
                const uint4 b = sr.v1 ? __ldg(reinterpret_cast<const uint4 *>(p1)) : make_uint4(0, 0, 0, 0);
                o0[0] = a.x; o0[1 % (GH / 2)] = a.y; o0[2 % (GH / 2)] = a.z; o0[3 % (GH / 2)] = a.w;
                o1[0] = b.x; o1[1 % (GH / 2)] = b.y; o1[2 % (GH / 2)] = b.z; o1[3 % (GH / 2)] = b.w;
            } else if (GH == 4) {
                const uint2 a = sr.v0 ? __ldg(reinterpret_cast<const uint2 *>(p0)) : make_uint2(0, 0);
                const uint2 b = sr.v1 ? __ldg(reinterpret_cast<const uint2 *>(p1)) : make_uint2(0, 0);
                o0[0] = a.x; o0[GH / 2 - 1] = a.y;
                o1[0] = b.x; o1[GH / 2 - 1] = b.y;
            } else {
                o0[0] = sr.v0 ? __ldg(reinterpret_cast<const uint32_t *>(p0)) : 0u;
                o1[0] = sr.v1 ? __ldg(reinterpret_cast<const uint32_t *>(p1)) : 0u;
            }
        };
        // per-stage bases: digit fragments [cs][q][half][lane][4] (q stride 256 words, cs
        // stride 256 G), factors [slot][G] (slot 2 cs + t/2)
        const int fstride = G * 256, cstride = 2 * G;
        const uint32_t *frag_lane = frag_s + lane * 4;
        const float *colf_tok = colf_s + (t >> 1) * G;
        const int *cfix_lane = cfix_s + 2 * t;          // [cs][q][8]: this thread's columns 2t, 2t+1
        uint32_t nx0[GH / 2], nx1[GH / 2];
        ScaleRows rows = scale_rows(u0 / C);
        load_scales(rows, (int)(u0 % C), nx0, nx1);
        int s = 0;
        uint32_t ph = 0;
        const uint8_t *stage = smem + L.stage_off;
        bool ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&bars->frag, 0, abort, err, kDevErrTimeout,
                                                                kWaitLimitNs));
        for (int64_t rb = u0 / C; rb * C < u1; rb++) {
            const int c_lo = (int)(rb == u0 / C ? u0 % C : 0);
            const int c_hi = (int)((rb + 1) * C <= u1 ? C : u1 - rb * C);
            float acc[CS][4];
#pragma unroll
            for (int cs = 0; cs < CS; cs++)
#pragma unroll
                for (int i = 0; i < 4; i++)
                    acc[cs][i] = 0.f;
            for (int c = c_lo; ok && c < c_hi; c++) {
                // this stage's scales were loaded one stage ago; start the next stage's now
                uint32_t sw0[GH / 2], sw1[GH / 2];
#pragma unroll
                for (int i = 0; i < GH / 2; i++) {
                    sw0[i] = nx0[i];
                    sw1[i] = nx1[i];
                }
                if (c + 1 < c_hi) {
                    load_scales(rows, c + 1, nx0, nx1);
                } else if ((rb + 1) * C < u1) {
                    rows = scale_rows(rb + 1);              // the next block's rows, once per block
                    load_scales(rows, 0, nx0, nx1);
                }
                // every lane observes the stage's phase itself; the verdict is made warp-uniform
                ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&bars->full[s], ph, abort, err,
                                                                    kDevErrTimeout, kWaitLimitNs));
                if (!ok)
                    break;                          // still meet the partner warp below
                const uint32_t *fb = frag_lane + c * (SC::kGroups * 256);
                const float *cb = colf_tok + c * SC::kGroups;
                const int *xb = cfix_lane + c * (SC::kGroups * 8);
                // groups expanded at once: four independent MMA chains at one column set, two
                // per column set beyond (fewer live A registers where there are more chains)
                constexpr int GPW = CS >= 2 || ROWS > 128 ? 2 : 4;
                constexpr int GP = GH < GPW ? GH : GPW;
#pragma unroll
                for (int h0 = 0; h0 < GH; h0 += GP) {          // GP groups at a time
                    uint32_t A[GP][4][4];                       // [group][mma][a0..a3]
#pragma unroll
                    for (int h = 0; h < GP; h++)
                        expand_group<FMT, SCH::kMask>(stage + woff[h0 + h][0], stage + woff[h0 + h][1], mul, A[h]);
                    if (h0 + GP == GH) {
                        __syncwarp();
                        if (lane == 0)
                            ptx::mbar_arrive(&bars->empty[s]);  // the stage's words are in registers
                    }
#pragma unroll
                    for (int cs = 0; cs < CS; cs++) {
                        int d[GP][4];
#pragma unroll
                        for (int h = 0; h < GP; h++) {          // GP independent chains
                            const uint32_t *fq = fb + cs * fstride + (h0 + h) * 256;
                            const uint4 bA = *reinterpret_cast<const uint4 *>(fq);
                            const uint4 bB = *reinterpret_cast<const uint4 *>(fq + 128);
                            // accumulator input of columns 2t, 2t+1 (both rows): 1.5 * 2^23 as float
                            // bits, minus 64 sum(d) for binary
                            if (SCH::kMask) {
                                const int2 cc = *reinterpret_cast<const int2 *>(xb + cs * G * 8 + (h0 + h) * 8);
                                const int cin[4] = {cc.x, cc.y, cc.x, cc.y};
                                mma_s8_first(d[h], A[h][0][0], A[h][0][1], A[h][0][2], A[h][0][3], bA.x, bA.y, cin);
                            } else {
                                mma_s8_first(d[h], A[h][0][0], A[h][0][1], A[h][0][2], A[h][0][3], bA.x, bA.y, magic);
                            }
                            mma_s8(d[h], A[h][1][0], A[h][1][1], A[h][1][2], A[h][1][3], bA.z, bA.w);
                            mma_s8(d[h], A[h][2][0], A[h][2][1], A[h][2][2], A[h][2][3], bB.x, bB.y);
                            mma_s8(d[h], A[h][3][0], A[h][3][1], A[h][3][2], A[h][3][3], bB.z, bB.w);
                        }
#pragma unroll
                        for (int h = 0; h < GP; h++) {
                            const __half2 p0 = *reinterpret_cast<const __half2 *>(&sw0[(h0 + h) >> 1]);
                            const __half2 p1 = *reinterpret_cast<const __half2 *>(&sw1[(h0 + h) >> 1]);
                            // 2^(e-27) of this quad-thread's token (2 cs + t/2) in this group, times the scales
                            const float f = cb[cs * cstride + h0 + h];
                            const float sf0 = ((h & 1) ? __high2float(p0) : __low2float(p0)) * f;
                            const float sf1 = ((h & 1) ? __high2float(p1) : __low2float(p1)) * f;
                            // exact int -> float: the accumulator started at the bits of 1.5 * 2^23
                            const float t0 = __int_as_float(d[h][0]) - 12582912.f;
                            const float t1 = __int_as_float(d[h][1]) - 12582912.f;
                            const float t2 = __int_as_float(d[h][2]) - 12582912.f;
                            const float t3 = __int_as_float(d[h][3]) - 12582912.f;
                            // (r0, col 2t) (r0, 2t+1) (r1, 2t) (r1, 2t+1): columns 2t, 2t+1 are digits of one token
                            acc[cs][0] = fmaf(t0, sf0, acc[cs][0]);
                            acc[cs][1] = fmaf(t1, sf0, acc[cs][1]);
                            acc[cs][2] = fmaf(t2, sf1, acc[cs][2]);
                            acc[cs][3] = fmaf(t3, sf1, acc[cs][3]);
                        }
                    }
                }
                stage += SC::kBytes;
                if (++s == S) {
                    s = 0;
                    ph ^= 1;
                    stage = smem + L.stage_off;
                }
            }

            // ---- the warp's accumulators go through its slot, where the digit columns of a
            // token (held by neighbouring quad-threads) are combined
            float *slot = red + (tile * 16) * (CS * 8);   // [16 rows][CS*8]
#pragma unroll
            for (int cs = 0; cs < CS; cs++) {
                slot[g8 * (CS * 8) + cs * 8 + 2 * t] = acc[cs][0];
                slot[g8 * (CS * 8) + cs * 8 + 2 * t + 1] = acc[cs][1];
                slot[(g8 + 8) * (CS * 8) + cs * 8 + 2 * t] = acc[cs][2];
                slot[(g8 + 8) * (CS * 8) + cs * 8 + 2 * t + 1] = acc[cs][3];
            }
            __syncwarp();
            if (!ok || *abort)
                break;
            // the tile's 16 M (row, token) sums, element e = lane + 32 i (16 M <= 128)
            float fin[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const int e = lane + 32 * i, rr = e / M, m = e % M;
                float v = 0.f;
                if (e < 16 * M) {
#pragma unroll
                    for (int dg = SCH::kCount - 1; dg >= 0; dg--)            // digit d weighs 2^(kBits d)
                        v = fmaf(v, (float)(1 << SCH::kBits), slot[rr * (CS * 8) + m * kColsPerTok + dg]);
                }
                fin[i] = v;
            }
            const int64_t row0 = rb * kRows + tile * 16;
            const bool whole = c_lo == 0 && c_hi == C;
            const int64_t x0 = rb * C, x1 = rb * C + C;     // owners of the block's first/last unit
            const int64_t i_first = (x0 + 1) * Pn / U + (((x0 + 1) * Pn) % U != 0) - 1;
            const int64_t i_last = x1 * Pn / U + ((x1 * Pn) % U != 0) - 1;
            const int nseg = (int)(i_last - i_first + 1);
            // a split block is the first (slot 0) or the last (slot 1) block of each CTA that
            // shares it; only its first owner can hold it in slot 1, and a CTA is the first
            // owner of at most one split block, so the counter is indexed by that owner
            const int end = rb == u0 / C ? 0 : 1;
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const int e = lane + 32 * i, rr = e / M, m = e % M;
                const int64_t n = row0 + rr;
                if (e < 16 * M) {
                    if (whole) {
                        if (n < N)
                            store_y<float>(y, yt, (int64_t)m * N + n, fin[i]);
                    } else {
                        part[(((int64_t)blockIdx.x * 2 + end) * kRows + tile * 16 + rr) * M + m] = fin[i];
                    }
                }
            }
            if (!whole) {
                // the last of the nseg warps that own these 16 rows sums the partials in
                // segment order; the counters were zeroed by this call's prep kernel. The warp
                // barrier orders every lane's partial stores before lane 0's release-add; lane
                // 0's acquire and the next warp barrier order the other segments' partials
                // before this warp's loads.
                __syncwarp();
                int last = 0;
                if (lane == 0)
                    last = ptx::atom_add_acq_rel_gpu(counters + i_first * kTiles + tile, 1u) == (unsigned)(nseg - 1);
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last) {
                    __syncwarp();
                    // element e = lane + 32 q of the tile's [16 rows][M] sums; the partials of
                    // eight segments are loaded at once (independent loads, one round trip),
                    // then added in segment order, so the result does not depend on timing
                    constexpr int QN = CS;                          // 16 M <= 32 CS elements
                    float v[QN];
#pragma unroll
                    for (int q = 0; q < QN; q++)
                        v[q] = 0.f;
                    for (int sg0 = 0; sg0 < nseg; sg0 += 8) {
                        float pv[8][QN];
#pragma unroll
                        for (int j = 0; j < 8; j++) {
                            const int sg = sg0 + j;
                            const int64_t i = i_first + sg;
                            const int slot_i = sg == 0 && i * U / Pn != x0 ? 1 : 0;
                            const float *pp = part + ((i * 2 + slot_i) * kRows + tile * 16) * M;
#pragma unroll
                            for (int q = 0; q < QN; q++) {
                                const int e = lane + 32 * q;
                                pv[j][q] = sg < nseg && e < 16 * M ? __ldcg(pp + e) : 0.f;
                            }
                        }
#pragma unroll
                        for (int j = 0; j < 8; j++)
#pragma unroll
                            for (int q = 0; q < QN; q++)
                                v[q] += pv[j][q];
                    }
#pragma unroll
                    for (int q = 0; q < QN; q++) {
                        const int e = lane + 32 * q, rr = e / M, m = e % M;
                        const int64_t n = row0 + rr;
                        if (e < 16 * M && n < N)
                            store_y<float>(y, yt, (int64_t)m * N + n, v[q]);
                    }
                }
            }
        }
    }
    if (threadIdx.x == 0) {
        // the fragment copy this thread issued must have landed before the CTA exits
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

int sm_count()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

struct Plan {
    int CS, stages, grid;
    int64_t NB, C, U;
    size_t part_bytes, counter_bytes, frag_bytes, colf_bytes, cfix_bytes;
    int n_counters;
};

template <int FMT, int CS>
int plan_stages(int G)
{
    for (int s = kMaxStages; s >= 2; s--)
        if (make_layout<FMT, CS, rows_for(FMT, CS)>(G, s).total <= kSmemLimit)
            return s;
    return 0;
}

int stages_for(int fmt, int CS, int G)
{
    if (fmt == BQ_BINARY_G128)
        return CS == 1 ? plan_stages<BQ_BINARY_G128, 1>(G) : CS == 2 ? plan_stages<BQ_BINARY_G128, 2>(G)
             : CS == 3 ? plan_stages<BQ_BINARY_G128, 3>(G) : plan_stages<BQ_BINARY_G128, 4>(G);
    return CS == 1 ? plan_stages<BQ_TERNARY_G128, 1>(G) : CS == 2 ? plan_stages<BQ_TERNARY_G128, 2>(G)
         : CS == 3 ? plan_stages<BQ_TERNARY_G128, 3>(G) : plan_stages<BQ_TERNARY_G128, 4>(G);
}

Plan make_plan(int M, int fmt, int64_t N, int64_t K)
{
    Plan p;
    p.CS = (M * kColsPerTok + 7) / 8;
    const int G = (int)(K / 128);
    p.stages = stages_for(fmt, p.CS, G);
    const int rows = rows_for(fmt, p.CS);
    p.NB = (N + rows - 1) / rows;
    p.C = K / (fmt == BQ_BINARY_G128 ? 1024 : 512);
    p.U = p.NB * p.C;
    const int64_t sms = sm_count();
    p.grid = (int)(p.U < sms ? p.U : sms);
    // partial sums: two block-sized slots per CTA (its first and last block, the only ones it
    // may share); one counter per tile of the split block each CTA opens
    auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
    p.part_bytes = al((size_t)p.grid * 2 * rows * M * 4);
    p.n_counters = p.grid * (rows / 16);
    p.counter_bytes = al((size_t)p.n_counters * 4);
    // the digit fragments and factors the prep kernel writes (the shared-memory images)
    p.frag_bytes = al((size_t)p.CS * G * 1024);
    p.colf_bytes = al((size_t)2 * p.CS * G * 4);
    p.cfix_bytes = al((size_t)p.CS * G * 32);
    return p;
}

template <int FMT, int CS, typename XT>
cudaError_t launch_tc_t(const GemvArgs &a, const Plan &pl, cudaStream_t s)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return cudaErrorNotSupported;
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    float *part = reinterpret_cast<float *>(ws);
    unsigned int *counters = reinterpret_cast<unsigned int *>(ws + pl.part_bytes);
    uint32_t *frag = reinterpret_cast<uint32_t *>(ws + pl.part_bytes + pl.counter_bytes);
    float *colf = reinterpret_cast<float *>(ws + pl.part_bytes + pl.counter_bytes + pl.frag_bytes);
    int *cfix = reinterpret_cast<int *>(ws + pl.part_bytes + pl.counter_bytes + pl.frag_bytes + pl.colf_bytes);

    CUtensorMap mw;
    const cuuint64_t wpr = (cuuint64_t)(FMT == BQ_BINARY_G128 ? a.K / 32 : a.K / 16);
    cuuint64_t wdims[2] = {wpr, (cuuint64_t)a.N};
    cuuint64_t wstr[1] = {wpr * 4};
    constexpr int ROWS = rows_for(FMT, CS);
    cuuint32_t wbox[2] = {32, (cuuint32_t)ROWS};         // 128 bytes x ROWS rows
    cuuint32_t est[2] = {1, 1};
    CUresult r = enc(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(a.words), wdims, wstr, wbox, est,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const cuuint64_t G = (cuuint64_t)(a.K / 128);
    const int smem = make_layout<FMT, CS, ROWS>((int)G, pl.stages).total;
    auto kern = gemv_tc_kernel<FMT, CS, ROWS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    // both kernels may start before their predecessor in the stream finishes (programmatic
    // dependent launch); each waits for it (griddepcontrol.wait) before touching its outputs
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t pcfg = {};
    const int items = (int)G * 2 * CS;
    pcfg.gridDim = dim3((unsigned)((items * 32 + kPrepThreads - 1) / kPrepThreads));
    pcfg.blockDim = dim3(kPrepThreads);
    pcfg.stream = s;
    pcfg.attrs = attr;
    pcfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&pcfg, gemv_prep_kernel<FMT, CS, XT>, static_cast<const XT *>(a.x), a.M, a.K, frag, colf,
                           cfix, counters, pl.n_counters);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(Geo<ROWS>::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mw, reinterpret_cast<const uint16_t *>(a.scales), a.M, a.N, a.K, a.y, a.yt, part, counters, frag, colf, cfix, pl.U, (int)pl.C, pl.stages, 1u,
                              a.dev_status);
}

template <int FMT, typename XT>
cudaError_t launch_tc_cs(const GemvArgs &a, const Plan &pl, cudaStream_t s)
{
    switch (pl.CS) {
    case 1: return launch_tc_t<FMT, 1, XT>(a, pl, s);
    case 2: return launch_tc_t<FMT, 2, XT>(a, pl, s);
    case 3: return launch_tc_t<FMT, 3, XT>(a, pl, s);
    default: return launch_tc_t<FMT, 4, XT>(a, pl, s);
    }
}

}  // namespace

// K a multiple of 1024 (whole 8-scale TMA boxes) and the digit fragments of all of K in
// shared memory next to at least two stages.
bool gemv_tc_supported(int M, int fmt, int64_t K)
{
    if (M < 1 || M > 8 || K % 1024 != 0)
        return false;
    return stages_for(fmt, (M * kColsPerTok + 7) / 8, (int)(K / 128)) >= 2;
}

size_t gemv_tc_workspace_bytes(int M, int fmt, int64_t N, int64_t K)
{
    Plan p = make_plan(M, fmt, N, K);
    return p.part_bytes + p.counter_bytes + p.frag_bytes + p.colf_bytes + p.cfix_bytes;
}

cudaError_t launch_gemv_tc(const GemvArgs &a, cudaStream_t s)
{
    Plan pl = make_plan(a.M, a.fmt, a.N, a.K);
    if (a.fmt == BQ_BINARY_G128)
        return a.xt == BQ_F16 ? launch_tc_cs<BQ_BINARY_G128, __half>(a, pl, s)
                              : launch_tc_cs<BQ_BINARY_G128, __nv_bfloat16>(a, pl, s);
    return a.xt == BQ_F16 ? launch_tc_cs<BQ_TERNARY_G128, __half>(a, pl, s)
                          : launch_tc_cs<BQ_TERNARY_G128, __nv_bfloat16>(a, pl, s);
}

// ---------------------------------------------------------------------------------------
// fixed scratch of bq_gemv_noalloc
// ---------------------------------------------------------------------------------------
// The workspace this kernel needs is at most two 128-row slots of M <= 8 fp32 partial sums
// per CTA, one counter per 16-row tile per CTA (the grid is at most one CTA per SM), and the
// digit fragments and factors, which fit in shared memory. This array holds that for grids of
// up to kStaticMaxCtas CTAs (1.56 MB). Nothing in it needs an initial value: each call's
// prep kernel zeroes the counters before the GEMV uses them.
constexpr int kStaticMaxCtas = 160;
// (rows x M of a slot: 128 x 8 at two to four column sets, 192 x 2 at one)
constexpr size_t kStaticPartBytes = (size_t)kStaticMaxCtas * 2 * 1024 * sizeof(float);
constexpr size_t kStaticCounterBytes = ((size_t)kStaticMaxCtas * kMaxTiles * 4 + 255) & ~size_t(255);
constexpr size_t kStaticFragBytes = (size_t)kSmemLimit;        // the fragments fit in shared memory
constexpr size_t kStaticColfBytes = ((size_t)kSmemLimit / 128 + 255) & ~size_t(255);
constexpr size_t kStaticCfixBytes = ((size_t)kSmemLimit / 32 + 255) & ~size_t(255);
static __device__ __align__(256) unsigned char
    g_gemv_scratch[kStaticPartBytes + kStaticCounterBytes + kStaticFragBytes + kStaticColfBytes + kStaticCfixBytes];

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
