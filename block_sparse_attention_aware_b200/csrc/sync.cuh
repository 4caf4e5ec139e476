// Bounded mbarrier waits shared by the warp-specialised kernels.  A wait that
// runs past its limit (WAIT_LIMIT_NS unless the kernel was given another)
// records FVATTN_ERR_TIMEOUT in the device status word and raises the CTA's
// abort flag, so every role leaves its loop, waits for its own copies and
// MMAs in flight, and the CTA still reaches its TMEM release.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace fv {

constexpr unsigned long long WAIT_LIMIT_NS = 4000000000ull;

// Returns false if the CTA aborted or the wait ran out.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned long long limit_ns = WAIT_LIMIT_NS) {
    if (mbar_try_wait(bar, parity)) return true;
    unsigned long long t0 = 0;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0u) {
            if (*abort_flag) return false;
            unsigned long long now = global_timer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > limit_ns) {
                record_status(FVATTN_ERR_TIMEOUT);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Warp-uniform variant: every lane waits, and the warp leaves together if
// any lane gave up (the .sync.aligned tcgen05 loads that follow need the
// whole warp).
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit_ns = WAIT_LIMIT_NS) {
    const bool ok = wait_bar(bar, parity, abort_flag, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

// Waits for two phases, trying both together until both have completed.
__device__ __forceinline__ bool wait_bar2(uint32_t bar1, uint32_t parity1, uint32_t bar2, uint32_t parity2,
                                          volatile int* abort_flag, unsigned long long limit_ns = WAIT_LIMIT_NS) {
    uint32_t done = mbar_try_wait2(bar1, parity1, bar2, parity2);
    if (done == 3u) return true;
    unsigned long long t0 = 0;
    for (uint32_t it = 1;; ++it) {
        if (done & 1u) {
            if (mbar_try_wait(bar2, parity2)) return true;
        } else if (done & 2u) {
            if (mbar_try_wait(bar1, parity1)) {
                done |= 1u;
                if (done == 3u) return true;
            }
        } else {
            done = mbar_try_wait2(bar1, parity1, bar2, parity2);
            if (done == 3u) return true;
        }
        if ((it & 255u) == 0u) {
            if (*abort_flag) return false;
            unsigned long long now = global_timer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > limit_ns) {
                record_status(FVATTN_ERR_TIMEOUT);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool wait_warp2(uint32_t bar1, uint32_t parity1, uint32_t bar2, uint32_t parity2,
                                           volatile int* abort_flag, unsigned long long limit_ns = WAIT_LIMIT_NS) {
    const bool ok = wait_bar2(bar1, parity1, bar2, parity2, abort_flag, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

// Drain wait used on the way out (ignores the abort flag): for copies or
// MMAs already issued, which complete on their own.
__device__ __forceinline__ bool wait_bar_drain(uint32_t bar, uint32_t parity,
                                               unsigned long long limit_ns = WAIT_LIMIT_NS) {
    unsigned long long t0 = 0;
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 255u) {
            unsigned long long now = global_timer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > limit_ns) {
                record_status(FVATTN_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

}  // namespace fv
