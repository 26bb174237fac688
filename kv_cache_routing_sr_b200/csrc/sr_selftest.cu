// Self-test of the bounded waits every kernel of this library relies on.
//
// All waits in the kernels (pipeline mbarriers, the routing kernel's staging
// copy) poll an mbarrier with try_wait and give up after a time bound read from
// %globaltimer, setting a device error bit instead of hanging. This kernel runs
// that mechanism on an mbarrier nothing ever arrives on, with a caller-given
// bound, and reports the outcome; the host checks that the wait ran out, took
// about the bound, and that the context is still usable afterwards. No fault,
// trap or unbounded loop is involved.
#include <cstdint>
#include <cuda_runtime.h>

#include "sinkrouter.h"
#include "sr_internal.h"
#include "sr_ptx.cuh"

namespace sr {
namespace {

__global__ void bounded_wait_selftest(uint64_t limit_ns, int32_t *status, unsigned long long *waited_ns)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1); // one arrival expected; none ever comes
        fence_mbar_init();
    }
    __syncthreads();
    const uint64_t t0 = global_timer_ns();
    bool done = false;
    while (!(done = mbar_try_wait(b, 0))) {
        if (global_timer_ns() - t0 > limit_ns)
            break;
    }
    const uint64_t t1 = global_timer_ns();
    if (threadIdx.x == 0) {
        *status = done ? 0 : SR_DEVERR_TIMEOUT;
        *waited_ns = (unsigned long long)(t1 - t0);
    }
}

} // namespace

cudaError_t launch_bounded_wait_selftest(int32_t limit_us, int32_t *status, unsigned long long *waited_ns,
                                         cudaStream_t stream)
{
    bounded_wait_selftest<<<1, 32, 0, stream>>>((uint64_t)limit_us * 1000ull, status, waited_ns);
    return cudaGetLastError();
}

} // namespace sr
