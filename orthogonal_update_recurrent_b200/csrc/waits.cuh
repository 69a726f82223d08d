// waits.cuh -- bounded device-side waits on mbarriers (sm_100a).
//
// Every wait of the tensor-core kernels on an mbarrier (a TMA copy landing, an MMA
// completing, a peer's partial result arriving) is bounded by the %globaltimer
// clock. A wait that runs out sets the CTA's abort flag and the library's device
// status word (read on the host by lattice_get_device_status, which reports
// LATTICE_ERR_TIMEOUT) and returns false, and the kernel then skips its remaining
// work instead of hanging the GPU. Two limits apply:
//   kTcWaitNs   any wait inside a kernel's main loop (after it, the kernel aborts);
//   kTcDrainNs  the exit drains, which keep a CTA alive until the asynchronous
//               copies and MMAs it issued have landed; these ignore the abort flag
//               and are longer, so that an abort never frees tensor memory or
//               retires a CTA under an operation still in flight.
#pragma once
#include <stdint.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace lattice {

constexpr uint64_t kTcWaitNs = 2000000000ull;   // 2 s bound on any single in-loop wait
constexpr uint64_t kTcDrainNs = 4000000000ull;  // 4 s bound on each exit drain

// Bounded wait: true when the phase completed; false (and the abort flag set)
// when the bound elapsed or another thread already aborted.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                        uint64_t limit_ns = kTcWaitNs) {
    if (ptx::mbar_try_wait(bar, parity)) return *abort == 0u;  // the common case: already complete
    if (*abort) return false;
    const uint64_t t0 = ptx::globaltimer();
    for (;;) {
        if (ptx::mbar_try_wait_sleep(bar, parity, 20000u)) return true;  // sleep <= 20 us per try
        if (*abort) return false;
        if (ptx::globaltimer() - t0 > limit_ns) {
            *abort = 1u;
            flag_timeout();
            return false;
        }
    }
}

// Warp-uniform form for the MMA warp: every lane waits, the warp agrees on the
// outcome (and is converged for the elect.sync issue that follows).
__device__ __forceinline__ bool tc_wait_warp(uint32_t bar, uint32_t parity, volatile uint32_t* abort) {
    const bool ok = tc_wait(bar, parity, abort);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool tc_live(volatile uint32_t* abort) {
    return __all_sync(0xffffffffu, *abort == 0u);
}

// Bounded wait that ignores the abort flag: used at exit so that no TMA write
// into shared memory is still in flight when the CTA retires.
__device__ __forceinline__ void tc_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer();
    for (;;) {
        if (ptx::mbar_try_wait_sleep(bar, parity, 20000u)) return;
        if (ptx::globaltimer() - t0 > kTcDrainNs) {
            flag_timeout();
            return;
        }
    }
}

}  // namespace lattice
