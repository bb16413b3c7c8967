// Placeholder for the tensor-core kernels while they are being brought up:
// reports them unsupported so that every request runs on the CUDA-core path.
#include "common.cuh"

namespace lsh {

bool hash_tc_supported(const Problem &) { return false; }
bool attn_tc_supported(const Problem &) { return false; }

cudaError_t launch_hash_tc(const Problem &, const void *, const void *, uint16_t *, uint32_t *, cudaStream_t)
{
    return cudaErrorNotSupported;
}
cudaError_t launch_attn_fwd_tc(const Problem &, const void *, const void *, const int32_t *, const float *,
                               __nv_bfloat16 *, float *, uint32_t *, cudaStream_t)
{
    return cudaErrorNotSupported;
}
cudaError_t launch_attn_bwd_tc(const Problem &, const void *, const void *, const void *, const int32_t *,
                               const float *, const float *, const float *, float *, float *, uint32_t *,
                               cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace lsh
