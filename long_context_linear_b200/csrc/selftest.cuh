// Self-test of the bounded-wait failure path: one CTA waits on an mbarrier
// that nothing will ever arrive on, gives up after `timeout_ns`, and records
// LA_ERR_TIMEOUT in the device status word, exactly as the compute kernels do
// when one of their waits runs out.  No fault, trap or hang is involved.
#pragma once
#include "sm100.cuh"

namespace lcl {
namespace selftest {

__global__ void wait_timeout_kernel(unsigned long long timeout_ns, int* status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(&bar, 0)) {
        if (globaltimer() - t0 > timeout_ns) {
            atomicExch(status, kStatusTimeout);
            break;
        }
    }
    // leave the barrier complete so the CTA exits with nothing pending on it
    mbar_arrive(&bar);
}

}  // namespace selftest
}  // namespace lcl
