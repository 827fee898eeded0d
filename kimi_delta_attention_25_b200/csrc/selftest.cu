// selftest.cu -- kda_selftest_wait_timeout: runs the bounded mbarrier wait that every kernel of the
// library uses, on a barrier that nothing arrives on, so that a test can watch it give up and report
// KDA_ERR_TIMEOUT through the workspace status word while the CUDA context stays usable.
#include <cuda_runtime.h>

#include "kda_internal.cuh"
#include "sm100.cuh"

namespace {

using namespace kda::sm100;

__global__ void wait_timeout_kernel(int32_t *status, long long budget)
{
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    // nothing arrives on `bar`: the wait runs out after `budget` cycles and records the timeout
    if (!mbar_wait(&bar, 0, budget)) kda::set_status(status, KDA_ERR_TIMEOUT);
}

bool aligned_to(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace

extern "C" kda_status_t kda_selftest_wait_timeout(void *workspace, size_t workspace_bytes,
                                                  long long budget_cycles, void *stream)
{
    if (!workspace || !aligned_to(workspace, 16) || workspace_bytes < kda::kStatusBytes)
        return KDA_ERR_INVALID_ARG;
    if (budget_cycles <= 0 || budget_cycles > KDA_SELFTEST_MAX_BUDGET) return KDA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(workspace, 0, kda::kStatusBytes, st) != cudaSuccess) return KDA_ERR_CUDA;
    wait_timeout_kernel<<<1, 32, 0, st>>>((int32_t *)workspace, budget_cycles);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
