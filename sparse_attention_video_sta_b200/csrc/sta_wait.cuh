// sta_wait.cuh -- bounded mbarrier waits shared by the STA kernels.  Every wait
// in a kernel has a time limit: when it runs out, the kernel records a timeout
// in the status word, raises the CTA's abort flag so the other roles stop too,
// drains what it issued and exits, leaving the context usable.
#pragma once

#include <stdint.h>

#include "sta_internal.h"
#include "sta_ptx.cuh"

namespace sta {

// Returns false when the CTA is aborting (another role gave up) or when this
// wait ran past `timeout_ns` (then it starts the abort).
__device__ __forceinline__ bool wait_bar_limited(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                 uint32_t* status, uint64_t timeout_ns) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    while (true) {
        for (int i = 0; i < 32; ++i)
            if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (ptx::globaltimer_ns() - t0 > timeout_ns) {
            *abort_flag = 1;
            atomicOr(status, kDevTimeout);
            return false;
        }
    }
}

// Drain wait used on the way out: bounded, never starts an abort.
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer_ns() - t0 > limit_ns) return;
    }
}

}  // namespace sta
