// bq_api.cu -- the C ABI of libbq: argument validation, dispatch to the kernels, status
// codes and the per-device error word.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "bq_internal.cuh"

namespace bq {

// Per-device status array: [kSlotErrBits] sticky device-side error bits,
// [kSlotInvalidCount] counter for the synchronous pack/unpack validation.
__device__ unsigned int g_status[4];

static thread_local char t_msg[512] = "no error";
static unsigned long long g_launches = 0;

// Test hooks (bq_debug_*): a shorter limit for the kernels' pipeline waits, and a number of
// compute calls that fail as if their launch had failed. BQ_FAULT=launch[:count] in the
// environment sets the latter when the library is loaded.
static uint64_t g_wait_ns = 0;
static int g_fail_launches = 0;

static int fault_from_env()
{
    const char *f = getenv("BQ_FAULT");
    if (!f || strncmp(f, "launch", 6) != 0)
        return 0;
    return f[6] == ':' ? atoi(f + 7) : 1;
}
[[maybe_unused]] static const int g_env_fault = (__atomic_store_n(&g_fail_launches, fault_from_env(), __ATOMIC_RELAXED), 0);

uint64_t pipeline_wait_ns()
{
    const uint64_t v = __atomic_load_n(&g_wait_ns, __ATOMIC_RELAXED);
    return v ? v : kWaitLimitDefaultNs;
}

bool take_injected_launch_failure()
{
    int n = __atomic_load_n(&g_fail_launches, __ATOMIC_RELAXED);
    while (n > 0)
        if (__atomic_compare_exchange_n(&g_fail_launches, &n, n - 1, false, __ATOMIC_RELAXED, __ATOMIC_RELAXED))
            return true;
    return false;
}

void note_launches(unsigned n) { __atomic_fetch_add(&g_launches, (unsigned long long)n, __ATOMIC_RELAXED); }

bq_status set_error(bq_status st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_msg, sizeof t_msg, fmt, ap);
    va_end(ap);
    return st;
}

bq_status check_launch(const char *what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return set_error(BQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return BQ_OK;
}

static constexpr int kMaxDevices = 64;
// Per-device cache of the architecture check and of the status array's device address,
// filled on the first call on each device under g_status_mu (host threads may make their
// first calls concurrently). The addresses belong to the device's primary context: after a
// cudaDeviceReset the library must be reloaded.
static std::mutex g_status_mu;
static unsigned int *g_status_ptr[kMaxDevices];
static bool g_checked_arch[kMaxDevices];

unsigned int *device_status(bq_status *st)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *st = set_error(BQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_checked_arch[dev]) {
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (major != 10 || minor != 0) {
            *st = set_error(BQ_ERR_UNSUPPORTED,
                            "device %d is sm_%d%d; libbq is built for sm_100a only", dev, major, minor);
            return nullptr;
        }
        g_checked_arch[dev] = true;
    }
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_status);
        if (e != cudaSuccess) {
            *st = set_error(BQ_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
            return nullptr;
        }
        g_status_ptr[dev] = static_cast<unsigned int *>(p);
    }
    *st = BQ_OK;
    return g_status_ptr[dev];
}

// The format and shape limits every call applies (no pointers looked at): what the size queries
// accept, so that they never plan for a shape the compute calls reject.
static bool shape_in_range(const bq_weight *w)
{
    return w && (w->fmt == BQ_BINARY_G128 || w->fmt == BQ_TERNARY_G128 || w->fmt == BQ_TERNARY_B3_G128) &&
           w->N >= 1 && w->N <= (int64_t(1) << 31) && w->K >= 128 && w->K <= (int64_t(1) << 24) && w->K % 128 == 0;
}

static bq_status validate_weight(const bq_weight *w)
{
    if (!w)
        return set_error(BQ_ERR_INVALID_ARG, "weight view is NULL");
    if (w->fmt != BQ_BINARY_G128 && w->fmt != BQ_TERNARY_G128 && w->fmt != BQ_TERNARY_B3_G128)
        return set_error(BQ_ERR_INVALID_ARG, "unknown format %d", (int)w->fmt);
    if (w->N < 1 || w->K < 128 || w->K % 128)
        return set_error(BQ_ERR_SHAPE, "N=%lld K=%lld: need N >= 1 and K a positive multiple of 128",
                         (long long)w->N, (long long)w->K);
    if (w->N > (int64_t(1) << 31) || w->K > (int64_t(1) << 24))
        return set_error(BQ_ERR_SHAPE, "N=%lld K=%lld beyond the supported range",
                         (long long)w->N, (long long)w->K);
    if (!w->words || !w->scales)
        return set_error(BQ_ERR_INVALID_ARG, "weight words or scales pointer is NULL");
    if (!aligned16(w->words) || !aligned16(w->scales))
        return set_error(BQ_ERR_ALIGNMENT, "weight words and scales must be 16-byte aligned");
    return BQ_OK;
}

}  // namespace bq

using namespace bq;

extern "C" {

const char *bq_version(void) { return "bq 0.1.0 sm_100a"; }

const char *bq_status_string(bq_status st)
{
    switch (st) {
    case BQ_OK: return "BQ_OK";
    case BQ_ERR_INVALID_ARG: return "BQ_ERR_INVALID_ARG";
    case BQ_ERR_SHAPE: return "BQ_ERR_SHAPE";
    case BQ_ERR_ALIGNMENT: return "BQ_ERR_ALIGNMENT";
    case BQ_ERR_DTYPE: return "BQ_ERR_DTYPE";
    case BQ_ERR_INVALID_CODE: return "BQ_ERR_INVALID_CODE";
    case BQ_ERR_CUDA: return "BQ_ERR_CUDA";
    case BQ_ERR_TIMEOUT: return "BQ_ERR_TIMEOUT";
    case BQ_ERR_UNSUPPORTED: return "BQ_ERR_UNSUPPORTED";
    case BQ_ERR_WORKSPACE: return "BQ_ERR_WORKSPACE";
    }
    return "unknown status";
}

const char *bq_last_error(void) { return t_msg; }

unsigned long long bq_kernel_launches(void) { return __atomic_load_n(&g_launches, __ATOMIC_RELAXED); }

size_t bq_packed_words(bq_format fmt, int64_t N, int64_t K)
{
    if (N < 1 || K < 128 || K % 128 || N > (int64_t(1) << 31) || K > (int64_t(1) << 24))
        return 0;
    if (fmt == BQ_BINARY_G128)
        return (size_t)N * (size_t)(K / 32);
    if (fmt == BQ_TERNARY_G128)
        return (size_t)N * (size_t)(K / 16);
    if (fmt == BQ_TERNARY_B3_G128)
        return (bq_packed_bytes(fmt, N, K) + 3) / 4;
    return 0;
}

size_t bq_packed_bytes(bq_format fmt, int64_t N, int64_t K)
{
    if (N < 1 || K < 128 || K % 128 || N > (int64_t(1) << 31) || K > (int64_t(1) << 24))
        return 0;
    if (fmt == BQ_TERNARY_B3_G128)
        return (size_t)N * (size_t)(26 * (K / 128));
    return 4 * bq_packed_words(fmt, N, K);
}

static bq_status pack_common(int fmt, const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                             void *words, uint16_t *s_out, cudaStream_t stream)
{
    if (!q || !s_in || !words || !s_out)
        return set_error(BQ_ERR_INVALID_ARG, "pack: NULL pointer");
    if (N < 1 || K < 128 || K % 128 || N > (int64_t(1) << 31) || K > (int64_t(1) << 24))
        return set_error(BQ_ERR_SHAPE, "pack: N=%lld K=%lld invalid", (long long)N, (long long)K);
    if (!aligned16(q) || !aligned16(words))
        return set_error(BQ_ERR_ALIGNMENT, "pack: q and words must be 16-byte aligned");
    if (take_injected_launch_failure())
        return set_error(BQ_ERR_CUDA, "%s: injected launch failure (test hook)", "pack");
    bq_status st;
    unsigned int *status = device_status(&st);
    if (!status)
        return st;
    unsigned int *cnt = status + kSlotInvalidCount;
    cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(unsigned int), stream);
    if (e == cudaSuccess)
        e = fmt == BQ_BINARY_G128    ? launch_pack_binary(q, N, K, static_cast<uint32_t *>(words), cnt, stream)
            : fmt == BQ_TERNARY_G128 ? launch_pack_ternary(q, N, K, static_cast<uint32_t *>(words), cnt, stream)
                                     : launch_pack_b3(q, N, K, static_cast<uint8_t *>(words), cnt, stream);
    if (e == cudaSuccess)
        note_launches(1);
    if (e == cudaSuccess && s_out != s_in)
        e = cudaMemcpyAsync(s_out, s_in, (size_t)N * (size_t)(K / 128) * 2, cudaMemcpyDeviceToDevice,
                            stream);
    unsigned int host_cnt = 0;
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(&host_cnt, cnt, sizeof host_cnt, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess)
        return set_error(BQ_ERR_CUDA, "pack: %s", cudaGetErrorString(e));
    if (host_cnt)
        return set_error(BQ_ERR_INVALID_CODE, "pack: %u weights outside the format's value set",
                         host_cnt);
    return BQ_OK;
}

bq_status bq_pack_binary_g128(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                              uint32_t *words, uint16_t *s_out, cudaStream_t stream)
{
    return pack_common(BQ_BINARY_G128, q, s_in, N, K, words, s_out, stream);
}

bq_status bq_pack_ternary_g128(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                               uint32_t *words, uint16_t *s_out, cudaStream_t stream)
{
    return pack_common(BQ_TERNARY_G128, q, s_in, N, K, words, s_out, stream);
}

bq_status bq_pack_ternary_b3_g128(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K, uint8_t *bytes,
                                  uint16_t *s_out, cudaStream_t stream)
{
    return pack_common(BQ_TERNARY_B3_G128, q, s_in, N, K, bytes, s_out, stream);
}

bq_status bq_quantize_g128(const void *w, bq_dtype wt, int64_t N, int64_t K, bq_format fmt, void *packed,
                           uint16_t *scales, cudaStream_t stream)
{
    if (!w || !packed || !scales)
        return set_error(BQ_ERR_INVALID_ARG, "quantize: NULL pointer");
    if (fmt != BQ_BINARY_G128 && fmt != BQ_TERNARY_G128 && fmt != BQ_TERNARY_B3_G128)
        return set_error(BQ_ERR_INVALID_ARG, "quantize: unknown format %d", (int)fmt);
    if (wt != BQ_F32 && wt != BQ_BF16 && wt != BQ_F16)
        return set_error(BQ_ERR_DTYPE, "quantize: w must be BQ_F32, BQ_BF16 or BQ_F16");
    if (N < 1 || K < 128 || K % 128 || N > (int64_t(1) << 31) || K > (int64_t(1) << 24))
        return set_error(BQ_ERR_SHAPE, "quantize: N=%lld K=%lld invalid", (long long)N, (long long)K);
    if (!aligned16(w) || !aligned16(packed) || !aligned16(scales))
        return set_error(BQ_ERR_ALIGNMENT, "quantize: w, packed and scales must be 16-byte aligned");
    if (take_injected_launch_failure())
        return set_error(BQ_ERR_CUDA, "%s: injected launch failure (test hook)", "quantize");
    bq_status st;
    if (!device_status(&st))
        return st;
    cudaError_t e = launch_quantize(fmt, w, wt, N, K, packed, scales, stream);
    if (e != cudaSuccess)
        return set_error(BQ_ERR_CUDA, "quantize launch: %s", cudaGetErrorString(e));
    note_launches(1);
    return BQ_OK;
}

bq_status bq_unpack_g128(const bq_weight *w, int8_t *q, uint16_t *s_out, cudaStream_t stream)
{
    bq_status st = validate_weight(w);
    if (st != BQ_OK)
        return st;
    if (!q)
        return set_error(BQ_ERR_INVALID_ARG, "unpack: q is NULL");
    if (!aligned16(q))
        return set_error(BQ_ERR_ALIGNMENT, "unpack: q must be 16-byte aligned");
    if (take_injected_launch_failure())
        return set_error(BQ_ERR_CUDA, "%s: injected launch failure (test hook)", "unpack");
    unsigned int *status = device_status(&st);
    if (!status)
        return st;
    unsigned int *cnt = status + kSlotInvalidCount;
    cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(unsigned int), stream);
    if (e == cudaSuccess)
        e = launch_unpack(w->fmt, w->words, w->N, w->K, q, cnt, stream);
    if (e == cudaSuccess)
        note_launches(1);
    if (e == cudaSuccess && s_out && s_out != w->scales)
        e = cudaMemcpyAsync(s_out, w->scales, (size_t)w->N * (size_t)(w->K / 128) * 2,
                            cudaMemcpyDeviceToDevice, stream);
    unsigned int host_cnt = 0;
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(&host_cnt, cnt, sizeof host_cnt, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess)
        return set_error(BQ_ERR_CUDA, "unpack: %s", cudaGetErrorString(e));
    if (host_cnt)
        return set_error(BQ_ERR_INVALID_CODE, "unpack: %u %s", host_cnt,
                         w->fmt == BQ_TERNARY_B3_G128 ? "bytes hold a value the base-3 encoding never writes"
                                                      : "ternary fields hold the invalid code 3");
    return BQ_OK;
}

static bq_status validate_xy(const char *who, const void *x, bq_dtype xt, const void *y, bq_dtype yt,
                             bool x_f32 = false)
{
    if (!x || !y)
        return set_error(BQ_ERR_INVALID_ARG, "%s: x or y is NULL", who);
    if (xt != BQ_F16 && xt != BQ_BF16 && !(x_f32 && xt == BQ_F32))
        return set_error(BQ_ERR_DTYPE, x_f32 ? "%s: x must be BQ_F16, BQ_BF16 or BQ_F32" : "%s: x must be BQ_F16 or BQ_BF16",
                         who);
    if (yt != BQ_F32 && yt != BQ_BF16 && yt != BQ_F16)
        return set_error(BQ_ERR_DTYPE, "%s: y must be BQ_F32, BQ_BF16 or BQ_F16", who);
    if (!aligned16(x) || !aligned16(y))
        return set_error(BQ_ERR_ALIGNMENT, "%s: x and y must be 16-byte aligned", who);
    return BQ_OK;
}

size_t bq_gemv_workspace_bytes(int64_t M, const bq_weight *w)
{
    if (!shape_in_range(w) || M < 1 || M > 8)
        return 0;
    return gemv_workspace_bytes((int)M, w->fmt, w->N, w->K);
}

bq_status bq_gemv(const void *x, bq_dtype xt, int64_t M, const bq_weight *w, void *y, bq_dtype yt,
                  void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    bq_status st = validate_weight(w);
    if (st != BQ_OK)
        return st;
    if ((st = validate_xy("gemv", x, xt, y, yt, true)) != BQ_OK)
        return st;
    if (M < 1 || M > 8)
        return set_error(BQ_ERR_SHAPE, "gemv: M=%lld, need 1 <= M <= 8", (long long)M);
    size_t need = gemv_workspace_bytes((int)M, w->fmt, w->N, w->K);
    if (need && (!workspace || ws_bytes < need))
        return set_error(BQ_ERR_WORKSPACE, "gemv: workspace needs %zu bytes, got %zu", need,
                         workspace ? ws_bytes : (size_t)0);
    if (workspace && !aligned16(workspace))
        return set_error(BQ_ERR_ALIGNMENT, "gemv: workspace must be 16-byte aligned");
    if (take_injected_launch_failure())
        return set_error(BQ_ERR_CUDA, "%s: injected launch failure (test hook)", "gemv");
    unsigned int *status = device_status(&st);
    if (!status)
        return st;
    GemvArgs a{x, (int)xt, (int)M, (int)w->fmt, w->N, w->K, w->words,
               reinterpret_cast<const __half *>(w->scales), y, (int)yt, workspace, ws_bytes, status,
               pipeline_wait_ns()};
    unsigned launches = 0;
    cudaError_t e = launch_gemv(a, stream, &launches);
    if (e != cudaSuccess)
        return set_error(BQ_ERR_CUDA, "gemv launch: %s", cudaGetErrorString(e));
    note_launches(launches);
    return BQ_OK;
}

bq_status bq_gemv_noalloc(const void *x, bq_dtype xt, int64_t M, const bq_weight *w, void *y,
                          bq_dtype yt, cudaStream_t stream)
{
    bq_status st = validate_weight(w);
    if (st != BQ_OK)
        return st;
    if ((st = validate_xy("gemv_noalloc", x, xt, y, yt, true)) != BQ_OK)
        return st;
    if (M < 1 || M > 8)
        return set_error(BQ_ERR_SHAPE, "gemv_noalloc: M=%lld, need 1 <= M <= 8", (long long)M);
    if (take_injected_launch_failure())
        return set_error(BQ_ERR_CUDA, "%s: injected launch failure (test hook)", "gemv_noalloc");
    unsigned int *status = device_status(&st);
    if (!status)
        return st;
    const size_t need = gemv_workspace_bytes((int)M, w->fmt, w->N, w->K);
    void *scratch = nullptr;
    size_t cap = 0;
    if (need) {
        cudaError_t e = gemv_static_scratch(&scratch, &cap);
        if (e != cudaSuccess)
            return set_error(BQ_ERR_CUDA, "gemv_noalloc: cudaGetSymbolAddress of the scratch array: %s",
                             cudaGetErrorString(e));
        if (need > cap)
            return set_error(BQ_ERR_WORKSPACE,
                             "gemv_noalloc: this shape on this device needs %zu bytes of scratch, more than "
                             "the %zu bytes of the library's fixed array; call bq_gemv with a workspace",
                             need, cap);
    }
    GemvArgs a{x, (int)xt, (int)M, (int)w->fmt, w->N, w->K, w->words,
               reinterpret_cast<const __half *>(w->scales), y, (int)yt, scratch, cap, status, pipeline_wait_ns()};
    unsigned launches = 0;
    cudaError_t e = launch_gemv(a, stream, &launches);
    if (e != cudaSuccess)
        return set_error(BQ_ERR_CUDA, "gemv_noalloc launch: %s", cudaGetErrorString(e));
    note_launches(launches);
    return BQ_OK;
}

size_t bq_gemv_topk_workspace_bytes(int64_t M, const bq_weight *w, int k)
{
    if (!shape_in_range(w) || M < 1 || M > 8 || k < 1 || k > 32)
        return 0;
    if (!gemv_rows_supported((int)M, w->fmt, w->N, w->K, k))
        return 0;
    return gemv_rows_workspace_bytes((int)M, w->fmt, w->N, w->K, k);
}

bq_status bq_gemv_topk(const void *x, bq_dtype xt, int64_t M, const bq_weight *w, int k, float *vals,
                       int32_t *idx, const float *u, float temperature, float top_p, int32_t *tokens,
                       void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    bq_status st = validate_weight(w);
    if (st != BQ_OK)
        return st;
    if (!x || !vals || !idx)
        return set_error(BQ_ERR_INVALID_ARG, "gemv_topk: x, vals or idx is NULL");
    if (xt != BQ_F16 && xt != BQ_BF16 && xt != BQ_F32)
        return set_error(BQ_ERR_DTYPE, "gemv_topk: x must be BQ_F16, BQ_BF16 or BQ_F32");
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(vals) & 3u) || (reinterpret_cast<uintptr_t>(idx) & 3u))
        return set_error(BQ_ERR_ALIGNMENT, "gemv_topk: x must be 16-byte aligned, vals and idx 4-byte aligned");
    if (M < 1 || M > 8)
        return set_error(BQ_ERR_SHAPE, "gemv_topk: M=%lld, need 1 <= M <= 8", (long long)M);
    if (k < 1 || k > 32 || k > w->N)
        return set_error(BQ_ERR_SHAPE, "gemv_topk: k=%d, need 1 <= k <= 32 and k <= N", k);
    if (u) {
        if (!tokens)
            return set_error(BQ_ERR_INVALID_ARG, "gemv_topk: u given without tokens");
        if ((reinterpret_cast<uintptr_t>(u) & 3u) || (reinterpret_cast<uintptr_t>(tokens) & 3u))
            return set_error(BQ_ERR_ALIGNMENT, "gemv_topk: u and tokens must be 4-byte aligned");
        if (!(temperature > 0.f) || !(temperature < 3.4e38f) || !(top_p > 0.f) || !(top_p <= 1.f))
            return set_error(BQ_ERR_INVALID_ARG, "gemv_topk: need temperature > 0 (finite) and 0 < top_p <= 1");
    }
    if (!gemv_rows_supported((int)M, w->fmt, w->N, w->K, k))
        return set_error(BQ_ERR_SHAPE,
                         "gemv_topk: needs K a multiple of 1024 and the digit fragments and logits of a CTA in "
                         "shared memory (K=%lld, N=%lld, M=%lld)",
                         (long long)w->K, (long long)w->N, (long long)M);
    const size_t need = gemv_rows_workspace_bytes((int)M, w->fmt, w->N, w->K, k);
    if (!workspace || ws_bytes < need)
        return set_error(BQ_ERR_WORKSPACE, "gemv_topk: workspace needs %zu bytes, got %zu", need,
                         workspace ? ws_bytes : (size_t)0);
    if (!aligned16(workspace))
        return set_error(BQ_ERR_ALIGNMENT, "gemv_topk: workspace must be 16-byte aligned");
    if (take_injected_launch_failure())
        return set_error(BQ_ERR_CUDA, "%s: injected launch failure (test hook)", "gemv_topk");
    unsigned int *status = device_status(&st);
    if (!status)
        return st;
    GemvArgs a{x, (int)xt, (int)M, (int)w->fmt, w->N, w->K, w->words,
               reinterpret_cast<const __half *>(w->scales), nullptr, (int)BQ_F32, workspace, ws_bytes, status,
               pipeline_wait_ns()};
    TopkArgs t{k, vals, idx, u, temperature, top_p, tokens};
    unsigned launches = 0;
    cudaError_t e = launch_gemv_topk(a, t, stream, &launches);
    if (e != cudaSuccess)
        return set_error(BQ_ERR_CUDA, "gemv_topk launch: %s", cudaGetErrorString(e));
    note_launches(launches);
    return BQ_OK;
}

// the workspace of bq_mlp_swiglu: the gate/up GEMV's x fragments, the fp32 activations a [M][F],
// the down GEMV's workspace (each part 256-byte aligned)
static size_t mlp_parts(int64_t M, const bq_weight *gate, const bq_weight *down, size_t *ws1, size_t *abytes)
{
    auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
    *ws1 = al(gemv_glu_workspace_bytes((int)M, gate->fmt, gate->N, gate->K));
    *abytes = al((size_t)M * (size_t)gate->N * 4);
    return *ws1 + *abytes + al(gemv_workspace_bytes((int)M, down->fmt, down->N, down->K));
}

static bq_status validate_mlp(int64_t M, const bq_weight *gate, const bq_weight *up, const bq_weight *down)
{
    bq_status st;
    if ((st = validate_weight(gate)) != BQ_OK || (st = validate_weight(up)) != BQ_OK ||
        (st = validate_weight(down)) != BQ_OK)
        return st;
    if (up->fmt != gate->fmt || up->N != gate->N || up->K != gate->K)
        return set_error(BQ_ERR_SHAPE, "mlp_swiglu: gate and up must have the same format and shape");
    if (down->K != gate->N)
        return set_error(BQ_ERR_SHAPE, "mlp_swiglu: down has K=%lld, gate and up N=%lld", (long long)down->K,
                         (long long)gate->N);
    if (M < 1 || M > 8)
        return set_error(BQ_ERR_SHAPE, "mlp_swiglu: M=%lld, need 1 <= M <= 8", (long long)M);
    if (!gemv_glu_supported((int)M, gate->fmt, gate->N, gate->K))
        return set_error(BQ_ERR_SHAPE, "mlp_swiglu: the gate/up projection needs K a multiple of 1024 and its x "
                                       "fragments in shared memory (K=%lld, M=%lld)", (long long)gate->K, (long long)M);
    return BQ_OK;
}

size_t bq_mlp_swiglu_workspace_bytes(int64_t M, const bq_weight *gate, const bq_weight *up, const bq_weight *down)
{
    if (!shape_in_range(gate) || !shape_in_range(up) || !shape_in_range(down) || M < 1 || M > 8 ||
        up->N != gate->N || up->K != gate->K || down->K != gate->N)
        return 0;
    if (!gemv_glu_supported((int)M, gate->fmt, gate->N, gate->K))
        return 0;
    size_t a, b;
    return mlp_parts(M, gate, down, &a, &b);
}

bq_status bq_mlp_swiglu(const void *x, bq_dtype xt, int64_t M, const bq_weight *gate, const bq_weight *up,
                        const bq_weight *down, void *y, bq_dtype yt, void *workspace, size_t ws_bytes,
                        cudaStream_t stream)
{
    bq_status st = validate_mlp(M, gate, up, down);
    if (st != BQ_OK)
        return st;
    if ((st = validate_xy("mlp_swiglu", x, xt, y, yt, true)) != BQ_OK)
        return st;
    size_t ws1, abytes;
    const size_t need = mlp_parts(M, gate, down, &ws1, &abytes);
    if (!workspace || ws_bytes < need)
        return set_error(BQ_ERR_WORKSPACE, "mlp_swiglu: workspace needs %zu bytes, got %zu", need,
                         workspace ? ws_bytes : (size_t)0);
    if (!aligned16(workspace))
        return set_error(BQ_ERR_ALIGNMENT, "mlp_swiglu: workspace must be 16-byte aligned");
    if (take_injected_launch_failure())
        return set_error(BQ_ERR_CUDA, "%s: injected launch failure (test hook)", "mlp_swiglu");
    unsigned int *status = device_status(&st);
    if (!status)
        return st;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *act = reinterpret_cast<float *>(ws + ws1);
    GemvArgs a1{x, (int)xt, (int)M, (int)gate->fmt, gate->N, gate->K, gate->words,
                reinterpret_cast<const __half *>(gate->scales), act, (int)BQ_F32, ws, ws1, status, pipeline_wait_ns()};
    unsigned l1 = 0, l2 = 0;
    cudaError_t e = launch_gemv_glu(a1, up->words, reinterpret_cast<const __half *>(up->scales), stream, &l1);
    if (e == cudaSuccess) {
        GemvArgs a2{act, (int)BQ_F32, (int)M, (int)down->fmt, down->N, down->K, down->words,
                    reinterpret_cast<const __half *>(down->scales), y, (int)yt, ws + ws1 + abytes,
                    ws_bytes - ws1 - abytes, status, pipeline_wait_ns()};
        e = launch_gemv(a2, stream, &l2);
    }
    if (e != cudaSuccess)
        return set_error(BQ_ERR_CUDA, "mlp_swiglu launch: %s", cudaGetErrorString(e));
    note_launches(l1 + l2);
    return BQ_OK;
}

size_t bq_gemm_prefill_workspace_bytes(int64_t M, const bq_weight *w)
{
    if (!shape_in_range(w) || M < 1 || M > (int64_t(1) << 24))
        return 0;
    return prefill_workspace_bytes(M, w->fmt, w->N, w->K);
}

bq_status bq_gemm_prefill(const void *x, bq_dtype xt, int64_t M, const bq_weight *w, void *y,
                          bq_dtype yt, void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    bq_status st = validate_weight(w);
    if (st != BQ_OK)
        return st;
    if ((st = validate_xy("gemm_prefill", x, xt, y, yt)) != BQ_OK)
        return st;
    if (M < 1 || M > (int64_t(1) << 24))
        return set_error(BQ_ERR_SHAPE, "gemm_prefill: M=%lld out of range", (long long)M);
    size_t need = prefill_workspace_bytes(M, w->fmt, w->N, w->K);
    if (need && (!workspace || ws_bytes < need))
        return set_error(BQ_ERR_WORKSPACE, "gemm_prefill: workspace needs %zu bytes", need);
    if (workspace && !aligned16(workspace))
        return set_error(BQ_ERR_ALIGNMENT, "gemm_prefill: workspace must be 16-byte aligned");
    if (take_injected_launch_failure())
        return set_error(BQ_ERR_CUDA, "%s: injected launch failure (test hook)", "gemm_prefill");
    unsigned int *status = device_status(&st);
    if (!status)
        return st;
    PrefillArgs a{x, (int)xt, M, (int)w->fmt, w->N, w->K, w->words,
                  reinterpret_cast<const __half *>(w->scales), y, (int)yt, need ? workspace : nullptr, status,
                  pipeline_wait_ns()};
    unsigned launches = 0;
    cudaError_t e = launch_prefill(a, stream, &launches);
    if (e != cudaSuccess)
        return set_error(BQ_ERR_CUDA, "gemm_prefill launch: %s", cudaGetErrorString(e));
    note_launches(launches);
    return BQ_OK;
}

bq_status bq_embed_gather(const int32_t *ids, int64_t T, const bq_weight *w, void *out, bq_dtype ot,
                          cudaStream_t stream)
{
    bq_status st = validate_weight(w);
    if (st != BQ_OK)
        return st;
    if (T < 0 || T > (int64_t(1) << 31))
        return set_error(BQ_ERR_SHAPE, "embed_gather: T=%lld out of range", (long long)T);
    if (T > 0 && (!ids || !out))
        return set_error(BQ_ERR_INVALID_ARG, "embed_gather: ids or out is NULL");
    if (ot != BQ_F32 && ot != BQ_BF16 && ot != BQ_F16)
        return set_error(BQ_ERR_DTYPE, "embed_gather: out must be BQ_F32, BQ_BF16 or BQ_F16");
    if (!aligned16(out))
        return set_error(BQ_ERR_ALIGNMENT, "embed_gather: out must be 16-byte aligned");
    if (take_injected_launch_failure())
        return set_error(BQ_ERR_CUDA, "%s: injected launch failure (test hook)", "embed_gather");
    unsigned int *status = device_status(&st);
    if (!status)
        return st;
    if (T == 0)
        return BQ_OK;
    cudaError_t e = launch_embed(w->fmt, ids, T, w->words, reinterpret_cast<const __half *>(w->scales),
                                 w->N, w->K, out, (int)ot, status, stream);
    if (e != cudaSuccess)
        return set_error(BQ_ERR_CUDA, "embed_gather launch: %s", cudaGetErrorString(e));
    note_launches(1);
    return BQ_OK;
}

void bq_debug_set_wait_limit_ns(uint64_t ns) { __atomic_store_n(&g_wait_ns, ns, __ATOMIC_RELAXED); }

void bq_debug_fail_next_launches(int count)
{
    __atomic_store_n(&g_fail_launches, count > 0 ? count : 0, __ATOMIC_RELAXED);
}

bq_status bq_get_device_error(cudaStream_t stream)
{
    bq_status st;
    unsigned int *status = device_status(&st);
    if (!status)
        return st;
    unsigned int bits = 0;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess)
        e = cudaMemcpy(&bits, status + kSlotErrBits, sizeof bits, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && bits)
        e = cudaMemset(status + kSlotErrBits, 0, sizeof bits);
    if (e != cudaSuccess)
        return set_error(BQ_ERR_CUDA, "get_device_error: %s", cudaGetErrorString(e));
    if (bits & kDevErrTimeout)
        return set_error(BQ_ERR_TIMEOUT, "a bounded device-side wait gave up");
    if (bits & kDevErrInvalidId)
        return set_error(BQ_ERR_INVALID_ARG, "an embedding id was outside [0, N)");
    return BQ_OK;
}

}  // extern "C"
