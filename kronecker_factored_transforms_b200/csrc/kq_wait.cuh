// kq_wait.cuh -- bounded mbarrier waits shared by the tcgen05 kernels.
//
// A wait gives up after `limit_ns` of %globaltimer time: it ORs the caller's
// site bit into the device status word `err`, raises the CTA's abort flag and
// returns false, so every role can leave its loop and the kernel returns
// instead of hanging.  kq_device_error reads and clears the status word.
#pragma once

#include <stdint.h>

#include "kq_tc05_ptx.cuh"

namespace kq {
namespace tc {

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // about one second

// Out of line: only reached when the phase is not complete at the first look.
__device__ __noinline__ inline bool wait_slow_err(uint32_t bar, uint32_t parity, volatile int *abort, unsigned site,
                                                  uint64_t limit_ns, bool ignore_abort, unsigned int *err) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 0) {
            if (!ignore_abort && *abort) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                atomicOr(err, site);
                *abort = 1;
                return false;
            }
        }
    }
}

// Wait for the phase of parity `parity` of mbarrier `bar` to complete, for at
// most `limit_ns`.  Returns false on timeout, or when another role already
// aborted (unless `ignore_abort`).
__device__ __forceinline__ bool wait_bounded_err(uint32_t bar, uint32_t parity, volatile int *abort, unsigned site,
                                                 uint64_t limit_ns, bool ignore_abort, unsigned int *err) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_slow_err(bar, parity, abort, site, limit_ns, ignore_abort, err);
}

// Position in a ring of n barrier-guarded slots: slot index and the parity of
// the slot's current phase; advancing past the last slot flips the parity.
struct Ring {
    uint32_t idx = 0, phase = 0;
    __device__ __forceinline__ void next(uint32_t n) {
        if (++idx == n) {
            idx = 0;
            phase ^= 1u;
        }
    }
};

}  // namespace tc
}  // namespace kq
