// waits.cuh -- bounded device waits shared by the warp-specialised kernels.
//
// Every wait gives up after a time bound (globaltimer), records
// MOE_ERR_TIMEOUT in the caller's status word and returns false, so a kernel
// never spins forever on a phase that will not complete.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace moeq4 {

constexpr unsigned long long kWaitNs = 2000000000ull;   // bound of every device wait (2 s)

__device__ __forceinline__ unsigned long long gtimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void wait_fail(int* status) { atomicCAS(status, 0, MOE_ERR_TIMEOUT); }

__device__ __forceinline__ bool wait_aborted(const int* status) {
    return ld_relaxed_s32(status) != 0;
}

// Wait on an mbarrier phase, bounded in time; gives up early when another
// thread has already recorded a failure.
__device__ __forceinline__ bool bounded_wait_bar(uint64_t* bar, uint32_t parity, int* status) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = gtimer_ns();
    for (unsigned it = 1;; it++) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31) == 0) {
            if (wait_aborted(status)) return false;
            if (gtimer_ns() - t0 > kWaitNs) { wait_fail(status); return false; }
        }
    }
}

}  // namespace moeq4
