// bq_internal.cuh -- declarations shared by libbq's translation units (product code only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "bq.h"

namespace bq {

// Bits of the per-device error word (device-side conditions, read by bq_get_device_error).
constexpr unsigned kDevErrInvalidId = 1u;   // embedding id outside [0, N)
constexpr unsigned kDevErrTimeout = 2u;     // a bounded wait gave up

// Slots of the per-device status array.
//   [0] sticky error bits (kDevErr*), [1] invalid-code counter used by pack/unpack.
constexpr int kSlotErrBits = 0;
constexpr int kSlotInvalidCount = 1;

// Per-device status array (device address, resolved once per device).
unsigned int *device_status(bq_status *st);

bq_status set_error(bq_status st, const char *fmt, ...);

// Limit of a bounded device-side wait: 2 s. Pipeline waits use the (test-only) shorter limit set
// by bq_debug_set_wait_limit_ns when there is one; the waits that drain copies and MMAs before a
// kernel exits always use this one.
constexpr uint64_t kWaitLimitDefaultNs = 2000000000ull;
uint64_t pipeline_wait_ns();
// True (once per injected failure) when a test asked the next launches to fail.
bool take_injected_launch_failure();

// Count of kernel launches enqueued by the library (instrumentation for benchmarks).
void note_launches(unsigned n);
bq_status check_launch(const char *what);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- launchers (each validates nothing; bq_api.cu validates before calling) ----

cudaError_t launch_pack_binary(const int8_t *q, int64_t N, int64_t K, uint32_t *words,
                               unsigned int *invalid_count, cudaStream_t s);
cudaError_t launch_pack_ternary(const int8_t *q, int64_t N, int64_t K, uint32_t *words,
                                unsigned int *invalid_count, cudaStream_t s);
cudaError_t launch_pack_b3(const int8_t *q, int64_t N, int64_t K, uint8_t *bytes, unsigned int *invalid_count,
                           cudaStream_t s);
cudaError_t launch_unpack(int fmt, const uint32_t *words, int64_t N, int64_t K, int8_t *q,
                          unsigned int *invalid_count, cudaStream_t s);

struct GemvArgs {
    const void *x;
    int xt;           // bq_dtype
    int M;
    int fmt;          // bq_format
    int64_t N, K;
    const uint32_t *words;
    const __half *scales;
    void *y;
    int yt;           // bq_dtype
    void *workspace;
    size_t ws_bytes;
    unsigned int *dev_status;
    uint64_t wait_ns;         // limit of the kernels' pipeline waits (bq_debug_set_wait_limit_ns)
};
size_t gemv_workspace_bytes(int M, int fmt, int64_t N, int64_t K);
cudaError_t launch_gemv(const GemvArgs &a, cudaStream_t s, unsigned *launches);
// integer tensor-core path, whole output rows per CTA (gemv_rows.cu): K a multiple of 1024 and
// the digit fragments of all of K in shared memory
bool gemv_rows_supported(int M, int fmt, int64_t N, int64_t K, int topk_k = 0);
size_t gemv_rows_workspace_bytes(int M, int fmt, int64_t N, int64_t K, int topk_k = 0);
cudaError_t launch_gemv_rows(const GemvArgs &a, cudaStream_t s, unsigned *launches);
// the same kernels selecting the k largest outputs of every token row (and drawing a token)
struct TopkArgs {
    int k;                    // 1 .. 32
    float *vals;              // [M][k]
    int *idx;                 // [M][k]
    const float *u;           // [M] or null
    float temperature, top_p;
    int *tokens;              // [M] (with u)
};
cudaError_t launch_gemv_topk(const GemvArgs &a, const TopkArgs &t, cudaStream_t s, unsigned *launches);
// the gate/up projection of a SwiGLU MLP: a.words / a.scales the gate rows, up_* the up rows (same
// format and shape); y[m][n] = silu(gate) * up
bool gemv_glu_supported(int M, int fmt, int64_t N, int64_t K);
size_t gemv_glu_workspace_bytes(int M, int fmt, int64_t N, int64_t K);
cudaError_t launch_gemv_glu(const GemvArgs &a, const uint32_t *up_words, const __half *up_scales, cudaStream_t s,
                            unsigned *launches);
// Device address and size of the fixed scratch array of bq_gemv_noalloc on the current
// device (gemv_rows.cu); resolved once per device.
cudaError_t gemv_static_scratch(void **ptr, size_t *bytes);

struct PrefillArgs {
    const void *x;
    int xt;
    int64_t M;
    int fmt;
    int64_t N, K;
    const uint32_t *words;
    const __half *scales;
    void *y;
    int yt;
    void *workspace;          // fp32 partials of split tail tiles (prefill_workspace_bytes)
    unsigned int *dev_status;
    uint64_t wait_ns;         // limit of the kernels' pipeline waits (bq_debug_set_wait_limit_ns)
};
size_t prefill_workspace_bytes(int64_t M, int fmt, int64_t N, int64_t K);
cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t s, unsigned *launches);

// least-squares fit of every group of 128 dense weights, packed (quantize.cu)
cudaError_t launch_quantize(int fmt, const void *w, int wt, int64_t N, int64_t K, void *packed, uint16_t *scales,
                            cudaStream_t s);

cudaError_t launch_embed(int fmt, const int32_t *ids, int64_t T, const uint32_t *words,
                         const __half *scales, int64_t N, int64_t K, void *out, int ot,
                         unsigned int *dev_status, cudaStream_t s);

// ---- small device helpers ----

template <int YT> struct OutT;
template <> struct OutT<BQ_F32> { using T = float; };
template <> struct OutT<BQ_BF16> { using T = __nv_bfloat16; };
template <> struct OutT<BQ_F16> { using T = __half; };

__device__ __forceinline__ void store_out(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ void store_out(__half *p, float v) { *p = __float2half_rn(v); }

__device__ __forceinline__ float load_x(const __half *p) { return __half2float(*p); }
__device__ __forceinline__ float load_x(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ float load_x(const float *p) { return *p; }

}  // namespace bq
