// Failure-detection self-test: exercises the bounded wait every pipeline kernel uses, on an
// mbarrier that nothing ever arrives on.  The wait gives up after `limit` cycles, latches
// MOE_ERR_DEVICE_TIMEOUT into the workspace status word and the kernel returns normally, so the
// CUDA context stays usable.  No trap, no fault, no unbounded loop.
#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

__global__ void wait_never_signalled(uint32_t* status, long long limit) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ volatile int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, status, 0x7E57, limit);
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int64_t limit_cycles,
                                                  void* stream) {
    using namespace moe;
    if (!workspace || workspace_bytes < kStatusWords * 4) return MOE_ERR_WORKSPACE;
    if (limit_cycles < 1 || limit_cycles > kWaitCycles) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* status = static_cast<uint32_t*>(workspace);
    if (cudaMemsetAsync(status, 0, kStatusWords * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    wait_never_signalled<<<1, 32, 0, s>>>(status, limit_cycles);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
