// Test hook for the error path of the time-bounded waits: one warp waits on an mbarrier
// that nothing will complete, gives up after the caller's limit, and reports
// ST_TIMEOUT through the status word, exactly as a pipeline stage whose copies never
// landed would.  Nothing faults and nothing hangs: the wait ends by its clock, the kernel
// returns, and the context stays usable.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace qkq {

namespace {

__global__ void k_bounded_wait_selftest(int *status, unsigned long long limit_ns)
{
    __shared__ uint64_t bar;
    const uint32_t b = smem_addr(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);  // one arrival expected; none will come
        fence_mbar_init();
    }
    __syncwarp();
    const bool done = __all_sync(FULL_MASK, mbar_wait_bounded(b, 0, limit_ns));
    if (!done && threadIdx.x == 0 && status != nullptr) atomicOr(status, ST_TIMEOUT);
}

}  // namespace

cudaError_t bounded_wait_selftest_launch(unsigned long long limit_ns, int *status,
                                         cudaStream_t stream)
{
    k_bounded_wait_selftest<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace qkq
