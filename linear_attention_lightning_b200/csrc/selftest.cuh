// Test hook for the failure-detection path: one CTA waits, with the bounded
// mbarrier wait every kernel of the library uses, on a barrier that nothing
// ever arrives on. The wait runs out, records LA_ERR_TIMEOUT in the device
// status word and returns, leaving the context usable.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace la {

__global__ void __launch_bounds__(32) selftest_wait_kernel() {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) ptx::mbar_wait(&bar, 0, &abort_flag);  // no arrival: runs out
}

}  // namespace la
