// Self-test of the bounded-wait path: one block waits on a shared-memory
// barrier that no thread or copy ever completes, gives up after `limit`
// polls and records the give-up in the workspace status word.  Nothing is in
// flight when it returns, so giving up is safe.
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

__global__ void selftest_wait_kernel(uint32_t *ctrl, uint32_t limit)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, limit))
        report_timeout(ctrl, kSiteSelftest);
}

}  // namespace

cudaError_t launch_selftest_wait(uint32_t *ctrl, uint32_t spin_limit, cudaStream_t st)
{
    selftest_wait_kernel<<<1, 32, 0, st>>>(ctrl, spin_limit);
    return cudaGetLastError();
}

}  // namespace ts
