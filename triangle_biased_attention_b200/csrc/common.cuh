// Shared device-side plumbing: the library's status word and bounded waits.
#pragma once

#include <cstdint>

#include "evo_attn.h"
#include "ptx_sm100.cuh"

namespace evo {

// Device status word of this library (one per device that loads it).  A
// kernel that gives up waiting records EVO_ERR_TIMEOUT here; the host reads
// and clears it in evo_attn_sync_status().
__device__ int g_status;

// A wait on an internal barrier longer than this is treated as a hang.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;


__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_status, 0, code); }

// Bounded wait with an explicit limit (the self-test uses a short one).
__device__ __noinline__ bool wait_bounded_for(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (ptx::globaltimer_ns() - t0 > limit_ns) {
            record_status(EVO_ERR_TIMEOUT);
            return false;
        }
    }
}

// Waits for the given phase parity of an mbarrier.  Returns false, after
// raising the CTA's abort flag and recording EVO_ERR_TIMEOUT, if the phase
// does not complete within kWaitTimeoutNs; returns false at once if another
// thread of the CTA has already raised the flag (pass abort_flag = nullptr to
// wait regardless of it, as the drain paths do).  One hardware-suspended
// try_wait first; past its suspension window the wait polls with
// non-blocking tests (measured faster than further suspended try_waits: the
// waiter resumes sooner once the phase completes), reading the flag and the
// clock every 32 polls.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint32_t flag = abort_flag != nullptr ? ptx::smem_u32(const_cast<int*>(abort_flag)) : 0u;
    const uint64_t t0 = ptx::globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (ptx::mbar_test_wait(bar, parity)) return true;
        if (flag != 0u) {
            int a;
            asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(a) : "r"(flag) : "memory");
            if (a) return false;
        }
        if (ptx::globaltimer_ns() - t0 > kWaitTimeoutNs) {
            if (abort_flag != nullptr) *abort_flag = 1;
            record_status(EVO_ERR_TIMEOUT);
            return false;
        }
    }
}

// Inline fast path: one non-blocking test (cheaper than a try_wait when the
// phase has already completed, the common case), then the bounded slow path.
__device__ __forceinline__ bool wait_fast(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (ptx::mbar_test_wait(bar, parity)) return true;
    return wait_bounded(bar, parity, abort_flag);
}

// Warp-uniform form: every lane waits (so every lane acquires the barrier),
// and the warp agrees on the outcome.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    const bool ok = wait_fast(bar, parity, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

}  // namespace evo
