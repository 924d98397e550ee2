// selftest.cuh -- self-test of the bounded waits and the device status word.
//
// Every pipeline wait in this library goes through mbar_wait_bounded: it
// gives up after kWaitBudgetNs of %globaltimer, sets its CTA's abort flag so
// the other roles stop waiting, and records kStatusTimeout with the waiting
// role in the device status word, which mxfp4_check_device_status reports as
// MXFP4_ERR_DEVICE_TIMEOUT.  This kernel makes that path run without a fault:
// thread 0 waits on an mbarrier that nothing arrives on; thread 32 starts
// 50 ms later on another such barrier, so thread 0's budget runs out first
// and its abort flag ends thread 32's wait without a second record.  Both
// waits end (by the budget, by the flag), so the kernel always returns.
#pragma once

#include "common.cuh"

namespace mxfp4 {
namespace selftest {

constexpr uint64_t kHeadStartNs = 50000000ull;

__global__ void __launch_bounds__(64) wait_timeout_kernel(uint32_t* status) {
    __shared__ uint64_t bars[2];
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(&bars[0], 0, &abort_flag, status, kRoleMma);
    if (threadIdx.x == 32) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < kHeadStartNs) {
        }
        mbar_wait_bounded(&bars[1], 0, &abort_flag, status, kRoleEpilogue);
    }
}

}  // namespace selftest
}  // namespace mxfp4
