// Self-test of the bounded device waits used by every tensor-core kernel: one
// CTA waits on an mbarrier that nothing ever completes.  The wait gives up
// after `budget` SM cycles, sets the timeout bit of the status word and the
// kernel returns normally, leaving the context usable.
#include "tc_common.cuh"

namespace lsh {

namespace {

__global__ void wait_selftest_kernel(uint32_t *__restrict__ status, long long budget)
{
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        abort = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)tc::mbar_wait(&bar, 0u, &abort, status, budget);
}

}  // namespace

cudaError_t launch_wait_selftest(uint32_t *status, long long budget, cudaStream_t st)
{
    wait_selftest_kernel<<<1, 32, 0, st>>>(status, budget);
    return cudaGetLastError();
}

}  // namespace lsh
