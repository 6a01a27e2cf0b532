// watchdog.cuh -- a self-test of the bounded waits that every pipeline kernel of the
// library uses (mbar_wait in sm100.cuh): a wait whose barrier never completes must give
// up after the wait limit, record STREAMKL_ERR_TIMEOUT in the device status word and raise
// the CTA's abort flag, and every other wait of the CTA must then give up early instead
// of running out its own limit.  Nothing here faults or traps: the kernel returns and the
// context stays usable.
#pragma once

#include "sm100.cuh"

namespace skl {

// [0] = bitmask of the waits that succeeded, [1], [2] = ns spent by waiter 0 and 1
__device__ unsigned long long g_watchdog[3];

// Delay before waiter 1 starts, so that an early exit of waiter 1 can only come from the
// abort flag raised by waiter 0.
constexpr unsigned long long kWatchdogStaggerNs = 500000000ull;

// One CTA of 64 threads.  Waiter w = lane 0 of warp w waits on barrier w (count 1).
// starve = 0: thread 33 arrives on both barriers before anyone waits; both waits succeed.
// starve != 0: nothing arrives.
__global__ void __launch_bounds__(64, 1) streamkl_watchdog_kernel(int starve) {
    __shared__ __align__(8) unsigned long long bars[2];
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (!starve && threadIdx.x == 33) {
        mbar_arrive(smem_u32(&bars[0]));
        mbar_arrive(smem_u32(&bars[1]));
    }
    __syncthreads();
    if (lane == 0) {
        if (warp == 1) {
            const unsigned long long s0 = globaltimer();
            while (globaltimer() - s0 < kWatchdogStaggerNs) {
            }
        }
        const unsigned long long t0 = globaltimer();
        const bool ok = mbar_wait(smem_u32(&bars[warp]), 0, &abort_flag);
        g_watchdog[1 + warp] = globaltimer() - t0;
        if (ok) atomicOr(&g_watchdog[0], 1ull << warp);
    }
}

}  // namespace skl
