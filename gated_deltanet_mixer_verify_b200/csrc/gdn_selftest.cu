// gdn_selftest.cu -- a test hook for the failure path shared by every kernel's bounded waits:
// a wait on an mbarrier that nothing completes must give up after its poll limit, report
// GDN_STATUS_WAIT_TIMEOUT in the caller's status word and return, leaving the context usable.
// Nothing here faults, traps or waits without a limit.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.cuh"

namespace gdn {
namespace {
using namespace dev;

__global__ void __launch_bounds__(32) gdn_bounded_wait_selftest_kernel(int32_t* status_word, uint32_t polls) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    // No thread ever arrives on `bar`: the same helper the kernels use must run out.
    const bool done = mbar_wait_bounded(&bar, 0, polls);
    if (!done && threadIdx.x == 0) atomicOr(status_word, kStatusWaitTimeout);
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int32_t* status_word, uint32_t polls, cudaStream_t stream) {
    gdn_bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(status_word, polls);
    return cudaGetLastError();
}

}  // namespace gdn
