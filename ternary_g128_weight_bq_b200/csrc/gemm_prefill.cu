// gemm_prefill.cu -- prefill GEMM on packed weights (tcgen05 path is added next).
#include "bq_internal.cuh"

namespace bq {

size_t prefill_workspace_bytes(int64_t M, int fmt, int64_t N, int64_t K)
{
    (void)M; (void)fmt; (void)N; (void)K;
    return 0;
}

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t s)
{
    (void)a; (void)s;
    return cudaErrorNotSupported;
}

}  // namespace bq
