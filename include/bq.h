/*
 * bq.h -- C ABI of libbq: linear layers run directly on packed binary-g128 and
 * ternary-g128 weights on an NVIDIA B200 (sm_100a). The weights are never expanded to a
 * dense FP16/BF16 tensor in device memory.
 *
 * The operations follow these pages:
 *   "prism-ml/Bonsai-27B-mlx-1bit - Hugging Face" model card
 *     - section "Weight representation: Binary g128": one sign bit per weight, bit 0 is
 *       -scale and bit 1 is +scale; 128 weights share one FP16 scale (1.125 bits/weight).
 *     - section "Highlights" / "Model overview": embedding, attention and MLP projections
 *       and the LM head are all binary-g128 layers.
 *     - section "CUDA (NVIDIA GPUs)": the matrix product unpacks the sign codes inside
 *       the kernel and applies the group scale; no dense FP16 copy is made.
 *     - section "Cross-platform throughput": tg128 (batch-1 decode) is bound by memory
 *       bandwidth, pp512 (512-token prompt) by compute.
 *   "Ternary Bonsai 27B vs ..." article (wmrh.cn), sections "三元量化技术突破" and
 *     "局限性与未来发展": ternary weights {-1, 0, +1} with the same FP16 scale per 128
 *     weights, kept in 2-bit storage.
 *
 * Packed layout (this library's fixed format; the pages give only the meaning of a
 * bit and the group size):
 *   - A weight matrix has N output rows and K inputs, K a multiple of 128; groups of 128
 *     run along K. Row-major over N with K inner.
 *   - Binary: uint32 words[N][K/32]; weight k of a row is bit (k % 32) of word (k / 32)
 *     (LSB first), so one group is 4 consecutive words (16 bytes).
 *   - Ternary: uint32 words[N][K/16]; weight k is the 2-bit field at bits
 *     2*(k % 16) .. 2*(k % 16)+1 of word (k / 16); code 0 -> -1, 1 -> 0, 2 -> +1, and code 3
 *     is invalid (never written by the pack calls; results of the compute calls are
 *     undefined where it occurs; bq_unpack_g128 reports it). One group is 8 words.
 *   - Ternary, base-3 storage (BQ_TERNARY_B3_G128; the article says the 2-bit storage is
 *     what ships today while the information is 1.71 bits per weight and native ternary
 *     kernels are in development): bytes[N][26 K/128]. Codes c = value + 1; bytes 0..23 of a
 *     group hold five codes each (group positions 5j .. 5j+4), bytes 24 and 25 four each
 *     (120..123, 124..127); a byte holding n codes stores ceil(256 v / 3^n), v the codes
 *     as a base-3 number with the first code most significant. A row is a run of blocks of
 *     8 groups (the last may hold fewer, nb): the 24 five-code bytes of each group of the
 *     block (group i at 24 i), then the two four-code bytes of each (at 24 nb + 2 i). With
 *     the scale this is 1.75 bits per weight. Byte values no v produces (13 of 256 for five
 *     codes, 175 for four) are invalid: never written by the pack call, undefined in the
 *     compute calls, reported by bq_unpack_g128.
 *   - Scales: IEEE binary16 scales[N][K/128].
 *   - Activations x[M][K] and outputs y[M][N] are dense row-major.
 *
 * Conventions for every call:
 *   - All data pointers are DEVICE pointers on the current CUDA device, owned by the
 *     caller; the library keeps no reference after the call returns. Pointers to words,
 *     scales, x, y, q and workspace must be 16-byte aligned.
 *   - Calls are asynchronous on `stream` unless stated otherwise. The returned status
 *     covers argument validation and the kernel launch; BQ_OK means "enqueued".
 *   - On any status other than BQ_OK nothing has been launched, and bq_last_error()
 *     returns a message for the calling thread.
 *   - Device-side conditions (an out-of-range token id, a bounded wait that gave up) set
 *     a per-device error word that bq_get_device_error() reads and clears.
 */
#ifndef BQ_H
#define BQ_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BQ_OK = 0,
    BQ_ERR_INVALID_ARG = 1,   /* null pointer, negative size or unknown enum value */
    BQ_ERR_SHAPE = 2,         /* K not a multiple of 128, M or N out of the supported range */
    BQ_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned */
    BQ_ERR_DTYPE = 4,         /* unsupported dtype for this argument */
    BQ_ERR_INVALID_CODE = 5,  /* a weight value outside the format's value set */
    BQ_ERR_CUDA = 6,          /* a CUDA runtime call or a launch failed */
    BQ_ERR_TIMEOUT = 7,       /* a bounded device-side wait gave up */
    BQ_ERR_UNSUPPORTED = 8,   /* the current device is not sm_100 */
    BQ_ERR_WORKSPACE = 9      /* workspace pointer null or smaller than required */
} bq_status;

/* The two *_INT_RANGE_ enumerators are not values to pass: they give the enum the range of a
 * 32-bit int, so that any int a caller passes is a representable value (the library rejects the
 * ones it does not know with BQ_ERR_INVALID_ARG or BQ_ERR_DTYPE) and reading it is defined
 * behaviour in C++ as well as in C. */
typedef enum {
    BQ_F16 = 0, BQ_BF16 = 1, BQ_F32 = 2,
    BQ_DTYPE_INT_RANGE_MIN_ = -2147483647 - 1, BQ_DTYPE_INT_RANGE_MAX_ = 2147483647
} bq_dtype;

typedef enum {
    BQ_BINARY_G128 = 0, BQ_TERNARY_G128 = 1, BQ_TERNARY_B3_G128 = 2,
    BQ_FORMAT_INT_RANGE_MIN_ = -2147483647 - 1, BQ_FORMAT_INT_RANGE_MAX_ = 2147483647
} bq_format;

/* Non-owning view of a packed weight matrix (device memory). Every call rejects a view outside
 * these limits with BQ_ERR_SHAPE, and every size query returns 0 for one. */
typedef struct {
    bq_format fmt;
    int64_t N;                /* output rows, 1 .. 2^31 */
    int64_t K;                /* inputs per row, a positive multiple of 128, at most 2^24 */
    const uint32_t *words;    /* [N][K/32] (binary), [N][K/16] (ternary), or the bytes
                                 [N][26 K/128] of the base-3 storage */
    const uint16_t *scales;   /* fp16 [N][K/128] */
} bq_weight;

/* Library version string, e.g. "bq 0.1.0 sm_100a". */
const char *bq_version(void);

/* Name of a status code. */
const char *bq_status_string(bq_status st);

/* Message describing the last non-OK status returned to the calling thread. */
const char *bq_last_error(void);

/* Total number of kernel launches this process has enqueued through libbq (all devices,
 * all threads); instrumentation for benchmarks. */
unsigned long long bq_kernel_launches(void);

/* Number of uint32 words in a packed matrix: N*K/32 (binary), N*K/16 (ternary) or the
 * base-3 bytes rounded up to whole words; 0 if the arguments are invalid. Scales always take
 * N*K/128 fp16 values. */
size_t bq_packed_words(bq_format fmt, int64_t N, int64_t K);

/* Bytes of a packed matrix: N*K/8, N*K/4, or N*26*K/128 (base-3); 0 if invalid. */
size_t bq_packed_bytes(bq_format fmt, int64_t N, int64_t K);

/*
 * Pack already-quantised weights into the binary-g128 format.
 *   q      int8 [N][K], values in {-1, +1} (-1 -> bit 0 -> -scale, +1 -> bit 1 -> +scale)
 *   s_in   fp16 [N][K/128] group scales; copied to s_out (s_out may equal s_in)
 *   words  out, uint32 [N][K/32]
 * Model card "prism-ml/Bonsai-27B-mlx-1bit", section "Weight representation: Binary g128".
 * SYNCHRONOUS: validates every q on the device, then waits for `stream`.
 * Returns BQ_ERR_INVALID_CODE if any q is outside {-1, +1} (words then hold garbage).
 */
bq_status bq_pack_binary_g128(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                              uint32_t *words, uint16_t *s_out, cudaStream_t stream);

/*
 * Pack already-quantised ternary weights (q in {-1, 0, +1}) into 2-bit codes
 * (code = q + 1), uint32 [N][K/16]. Ternary Bonsai 27B article (wmrh.cn), section
 * "局限性与未来发展" (2-bit storage). Synchronous, like the binary call; returns
 * BQ_ERR_INVALID_CODE if any q is outside {-1, 0, +1}.
 */
bq_status bq_pack_ternary_g128(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                               uint32_t *words, uint16_t *s_out, cudaStream_t stream);

/*
 * Pack already-quantised ternary weights (q in {-1, 0, +1}) into the base-3 storage
 * described at the top of this file, bytes [N][26 K/128] (16-byte aligned). Ternary Bonsai
 * 27B article (wmrh.cn), section "局限性与未来发展" (1.71 bits per weight in principle;
 * native ternary kernels in development). Synchronous, like the other pack calls; returns
 * BQ_ERR_INVALID_CODE if any q is outside {-1, 0, +1}.
 */
bq_status bq_pack_ternary_b3_g128(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                                  uint8_t *bytes, uint16_t *s_out, cudaStream_t stream);

/*
 * Dense weights to a packed format: the least-squares fit of every group of 128 weights w,
 * packed as the pack calls do. The pages give the formats but not how q and s are obtained
 * (model card section "Weight representation: Binary g128" refers to a whitepaper that is not
 * among them); this call takes
 *   binary:  q = +1 where w >= 0, else -1; s = mean |w| (the best scale for those signs);
 *   ternary (2-bit or base-3 storage): the q in {-1, 0, +1} and s minimising sum (w - s q)^2,
 *            i.e. q = sign(w) on the j largest |w| (equal |w|: lower position first) with j
 *            maximising (their sum)^2 / j (the smallest such j; none for a group of zeros),
 *            and s their mean |w|;
 * s rounded to fp16 (nearest even). Sums and scores are taken in fp64.
 *   w       [N][K] dense, wt = BQ_F32, BQ_BF16 or BQ_F16 (infinities or NaNs give undefined codes)
 *   packed  out: uint32 words [N][K/32] or [N][K/16], or bytes [N][26 K/128] (base-3)
 *   scales  out: fp16 [N][K/128]
 * Asynchronous on `stream` (one kernel); all pointers 16-byte aligned.
 */
bq_status bq_quantize_g128(const void *w, bq_dtype wt, int64_t N, int64_t K, bq_format fmt,
                           void *packed, uint16_t *scales, cudaStream_t stream);

/*
 * Inverse of the pack calls: q int8 [N][K] and, if s_out is not NULL, a copy of the
 * scales. SYNCHRONOUS. Returns BQ_ERR_INVALID_CODE if a ternary code 3, or an invalid base-3
 * byte, is found (the q of its codes is written as 0).
 */
bq_status bq_unpack_g128(const bq_weight *w, int8_t *q, uint16_t *s_out, cudaStream_t stream);

/*
 * Decode GEMV: y[m][n] = sum_g s[n][g] * sum_{k in group g} v[n][k] * x[m][k], with
 * v = 2b - 1 (binary) or c - 1 (ternary, 2-bit or base-3 storage), for M <= 8 token rows.
 * Model card "prism-ml/Bonsai-27B-mlx-1bit", sections "Weight representation: Binary g128"
 * and "CUDA (NVIDIA GPUs)"; the decode (tg128) workload of section "Cross-platform
 * throughput".
 *   x          [M][K], xt = BQ_F16, BQ_BF16 or BQ_F32. A token row that holds an infinity or a NaN
 *              gets non-finite outputs (NaN where K is a multiple of 1024, where the kernels
 *              carry x as integer digits per group; +-inf or NaN otherwise).
 *   M          1..8
 *   y          [M][N], yt = BQ_F32, BQ_BF16 or BQ_F16 (fp32 accumulation, rounded once)
 *   workspace  device scratch of at least bq_gemv_workspace_bytes(M, w) bytes (may be
 *              NULL when that size is 0): the digit fragments of x that a prep kernel writes
 *              once per call (1 KB per 128 inputs and per two tokens, plus factors). Its
 *              contents need not be initialised and are left undefined. Calls that share a
 *              workspace must be ordered on one stream.
 * Launches: two kernels (the prep and the GEMV, both programmatic dependent launches) when K
 * is a multiple of 1024 and the fragments fit in shared memory (K <= 5120 at M = 8, K <= 20480
 * at M = 1); otherwise one SIMT kernel. Base-3 weights are decoded inside the same kernels.
 */
bq_status bq_gemv(const void *x, bq_dtype xt, int64_t M, const bq_weight *w,
                  void *y, bq_dtype yt, void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes bq_gemv needs for this shape (0 if none). */
size_t bq_gemv_workspace_bytes(int64_t M, const bq_weight *w);

/*
 * bq_gemv without a workspace argument: the same product, same kernels, same arguments and
 * results, with the scratch taken from a fixed array inside the library. It allocates no
 * device memory. The model card and the Ternary Bonsai article have no counterpart: this
 * call exists for callers that cannot allocate device memory per call, or do not want to:
 *   - code that already handed all free device memory to its own pools (weights, KV cache)
 *     and has no allocator to draw a workspace from;
 *   - a decode loop that must not call cudaMalloc or cudaFree between steps, since those
 *     calls can synchronise the device and stall the queued work;
 *   - plain C hosts that do not want to size, own and free a buffer per weight shape.
 * Limit: the array is 256 KB per device. It holds the digit fragments of x that this GEMV
 * keeps in scratch, which by construction fit in one CTA's shared memory, so every shape the
 * tensor-core path takes fits; a shape that needs more returns BQ_ERR_WORKSPACE with the two
 * sizes in bq_last_error(), and bq_gemv with a workspace then serves it.
 * Set-up: the first call on each device (with that device current) resolves the array's
 * address; make that first call before any stream capture. Later calls do no set-up.
 * Sharing: all calls on a device share the one array. Nothing in it needs an initial value
 * (each call zeroes the counters it uses before using them). Calls that may overlap
 * on the device (different streams, several host threads) race on the array and give wrong
 * results: order them on one stream, or use bq_gemv with a workspace per stream.
 * Errors: as bq_gemv, plus BQ_ERR_WORKSPACE for the limit above.
 */
bq_status bq_gemv_noalloc(const void *x, bq_dtype xt, int64_t M, const bq_weight *w,
                          void *y, bq_dtype yt, cudaStream_t stream);

/*
 * LM head with top-k: the decode GEMV's outputs y[m][n] (as bq_gemv computes them, fp32) are
 * not written; instead each token row's k largest are returned, and optionally a token drawn
 * from them. Model card "prism-ml/Bonsai-27B-mlx-1bit", section "Generation parameters":
 * top-k 20, top-p 0.95, temperature 0.7 (the pages do not give the order of the three; this
 * call applies them as described for `tokens` below).
 *   x, xt, M, w  as bq_gemv (M 1..8); w->K a multiple of 1024 (the tensor-core path).
 *   k            1..32 and k <= N.
 *   vals, idx    out, float [M][k] and int32 [M][k]: the k largest outputs of each row in
 *                descending order (equal values: lower index first) and their row indices n.
 *   u            NULL, or float [M] uniform numbers in [0, 1), one per token row (device).
 *   temperature, top_p   used with u: temperature > 0, 0 < top_p <= 1.
 *   tokens       out with u, int32 [M]: probabilities softmax(v / temperature) over the k
 *                candidates; the shortest leading run of candidates whose probabilities sum
 *                to at least top_p is kept; the token is the first kept candidate whose
 *                cumulative probability, renormalised over the kept ones, exceeds u.
 *   workspace    bq_gemv_topk_workspace_bytes(M, w, k) bytes (16-byte aligned): the digit
 *                fragments of x, each CTA's k candidates per row and a ticket counter. Contents
 *                need not be initialised; calls sharing a workspace must be ordered on one stream.
 * The GEMV's CTAs each own whole rows: a CTA keeps its rows' outputs in shared memory, selects
 * their k largest and writes them to the workspace; the last CTA to finish selects the k
 * largest of those and writes vals, idx and tokens. x with an infinity or NaN gives an
 * unspecified selection for that row.
 * Errors: as bq_gemv; BQ_ERR_SHAPE for K not a multiple of 1024 or a k out of range.
 * Launches: two kernels (the x prep and the GEMV with the selection).
 */
bq_status bq_gemv_topk(const void *x, bq_dtype xt, int64_t M, const bq_weight *w, int k,
                       float *vals, int32_t *idx, const float *u, float temperature, float top_p,
                       int32_t *tokens, void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes bq_gemv_topk needs (0 if the shape or k is not supported). */
size_t bq_gemv_topk_workspace_bytes(int64_t M, const bq_weight *w, int k);

/*
 * SwiGLU MLP of a decode step: y = (silu(x Wg^T) * (x Wu^T)) Wd^T with silu(z) = z / (1 + e^-z).
 * Model card "prism-ml/Bonsai-27B-mlx-1bit", section "Model overview": the blocks use a SwiGLU
 * MLP. The gate and up projections run as one GEMV over interleaved 16-row tiles of gate and up,
 * whose epilogue writes the activations a = silu(g) * u (fp32, in the workspace) instead of g and
 * u; the down GEMV then reads a as its x. Three kernel launches (the x prep, the gate/up GEMV,
 * the down GEMV's prep and GEMV: four) chained by programmatic dependent launch.
 *   x       [M][K], xt = BQ_F16, BQ_BF16 or BQ_F32; M 1..8
 *   gate, up  the same format, N = F rows, K a multiple of 1024
 *   down    N rows, K = F (any format)
 *   y       [M][N], yt = BQ_F32, BQ_BF16 or BQ_F16
 *   workspace  bq_mlp_swiglu_workspace_bytes(M, gate, up, down) bytes, 16-byte aligned: the x
 *           fragments of the gate/up GEMV, a (M*F*4 bytes) and the down GEMV's workspace.
 * Errors: as bq_gemv; BQ_ERR_SHAPE when the shapes do not chain or the gate/up projection does not
 * fit the tensor-core path.
 */
bq_status bq_mlp_swiglu(const void *x, bq_dtype xt, int64_t M, const bq_weight *gate,
                        const bq_weight *up, const bq_weight *down, void *y, bq_dtype yt,
                        void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes bq_mlp_swiglu needs (0 if the shapes are not supported). */
size_t bq_mlp_swiglu_workspace_bytes(int64_t M, const bq_weight *gate, const bq_weight *up,
                                     const bq_weight *down);

/*
 * Prefill GEMM: the same product for M up to 512 token rows (larger M is accepted),
 * Y[M][N] = X[M][K] * W^T with W the dequantised +-s (binary) or {-s, 0, +s} (ternary,
 * 2-bit or base-3 storage) matrix. The packed bits are expanded on chip, straight into tensor memory, as the A
 * operand of the tensor cores (tcgen05, accumulation in fp32 in tensor memory); no expanded
 * copy is written to device memory. The pp512 (512-token prompt, compute-bound) workload of
 * the model card's section "Cross-platform throughput" and of the Ternary Bonsai 27B
 * article's throughput table.
 *   x  [M][K], xt = BQ_F16 or BQ_BF16. The tensor-core operands are always fp16: the weight
 *      operand is +-s (or 0) in fp16, which holds every fp16 scale exactly. fp16 x is used as
 *      it is. bf16 x is first copied into the workspace as fp16 x * 2^e, with one power of two
 *      per token row that puts the row's largest finite |x| in [2^14, 2^15); the fp32 results
 *      are multiplied by 2^-e (exact). Every bf16 element within a factor 2^31 of its row's
 *      largest magnitude is carried exactly; smaller ones are rounded to fp16's subnormal
 *      spacing, an error of at most 2^-39 of the row's largest magnitude. Infinities and NaNs
 *      stay non-finite.
 *   y  [M][N], yt = BQ_F32, BQ_BF16 or BQ_F16.
 *   workspace: at least bq_gemm_prefill_workspace_bytes(M, w) bytes, 16-byte aligned. It holds
 *      the fp16 copy of bf16 x (M*K*2 bytes, reserved for either x type) with its M factors,
 *      and fp32 partial sums when the last wave of output tiles would leave most SMs idle and
 *      its tiles are split along K instead (for example M = 512, N = 20480: 18.9 MB of
 *      partials). Contents need not be initialised; calls that share a workspace must be
 *      ordered on one stream.
 * Launches: one kernel, plus the conversion pass for bf16 x, plus two (the split grid and a
 * reduce pass) when the tail of the output tiles is split along K.
 */
bq_status bq_gemm_prefill(const void *x, bq_dtype xt, int64_t M, const bq_weight *w,
                          void *y, bq_dtype yt, void *workspace, size_t ws_bytes,
                          cudaStream_t stream);

size_t bq_gemm_prefill_workspace_bytes(int64_t M, const bq_weight *w);

/*
 * Embedding lookup on a packed matrix: out[t][k] = s[id][k/128] * v[id][k] for
 * id = ids[t]. Model card section "Highlights": the embedding is one of the binary layers.
 *   ids  int32 [T] device array
 *   out  [T][K], ot = BQ_BF16 (the +-s value rounded to nearest even), BQ_F16 (exact) or
 *        BQ_F32 (exact)
 * An id outside [0, N) is not read: its row is written as zeros and the device error
 * word records BQ_ERR_INVALID_ARG (see bq_get_device_error).
 */
bq_status bq_embed_gather(const int32_t *ids, int64_t T, const bq_weight *w, void *out,
                          bq_dtype ot, cudaStream_t stream);

/*
 * Wait for `stream`, then read and clear the current device's error word. Returns BQ_OK,
 * BQ_ERR_INVALID_ARG (an out-of-range embedding id was seen) or BQ_ERR_TIMEOUT (a bounded
 * device wait gave up; that kernel's outputs are undefined). Kernels on any stream of
 * the device share the word.
 */
bq_status bq_get_device_error(cudaStream_t stream);

/*
 * Test hooks for the failure paths (not for production use; process-wide, any thread).
 *
 * bq_debug_set_wait_limit_ns: the pipeline waits of the GEMV and prefill kernels (a stage of
 * weights or x to arrive, a slot to free, the accumulator to complete) give up after `ns`
 * nanoseconds instead of the built-in 2 s; 0 restores 2 s. Below 1000 ns (finer than the
 * device timer) a wait gives up at its first poll that finds the phase incomplete, which makes
 * a timeout certain on any call that waits for a copy. A wait that gives up records
 * BQ_ERR_TIMEOUT in the device error word (see bq_get_device_error); the kernel then skips its
 * remaining work, waits (2 s at most) for its copies and MMAs in flight, frees its tensor
 * memory and returns, and that call's outputs are undefined. Later calls are unaffected.
 *
 * bq_debug_fail_next_launches: the next `count` compute calls (pack, unpack, gemv,
 * gemv_noalloc, gemm_prefill, embed_gather) that pass argument validation return BQ_ERR_CUDA
 * ("injected launch failure") without launching anything, as if their launch had failed.
 * BQ_FAULT=launch or BQ_FAULT=launch:<count> in the environment sets the same when the library
 * is loaded. 0 cancels.
 */
void bq_debug_set_wait_limit_ns(uint64_t ns);
void bq_debug_fail_next_launches(int count);

#ifdef __cplusplus
}
#endif

#endif /* BQ_H */
