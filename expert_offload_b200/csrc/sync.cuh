// sync.cuh - bounded waits of the persistent kernels.  Every spin ends: when
// the condition holds, when this CTA's abort flag is set, when another CTA has
// written an error into the status word, or at a deadline on %globaltimer,
// after which HFQ_ERR_TIMEOUT is recorded in the status word.
#pragma once

#include <cstdint>

#include "common.h"
#include "ptx.cuh"

namespace hfq {

struct WaitCtx {
    unsigned *status;         // workspace status word (0 = ok)
    long long timeout_ns;
    volatile int *abort;      // this CTA's abort flag (shared memory)
};

__device__ __forceinline__ bool deadline_passed(uint64_t t0, long long timeout_ns)
{
    return (long long)(globaltimer_ns() - t0) > timeout_ns;
}

__device__ __forceinline__ void raise_timeout(const WaitCtx &w)
{
    *w.abort = 1;
    atomicCAS(w.status, 0u, (unsigned)HFQ_ERR_TIMEOUT);
}

// Waits until *p >= target (acquire, gpu scope).  The clock is read only once
// the wait has not completed after 64 polls.
__device__ inline bool wait_counter_ge(const WaitCtx &w, const unsigned *p, unsigned target)
{
    uint64_t t0 = 0;
    for (int it = 0;; ++it) {
        if (ld_acquire_gpu(p) >= target) return true;
        if (*w.abort) return false;
        if (it == 64) t0 = globaltimer_ns();
        if (it > 64 && (it & 63) == 0) {
            if (*(volatile unsigned *)w.status != 0u) { *w.abort = 1; return false; }
            if (deadline_passed(t0, w.timeout_ns)) { raise_timeout(w); return false; }
        }
        if (it > 16) __nanosleep(32);
    }
}

// Waits until the producer has armed use `seq` of a ring stage (*armed ==
// seq), so that a following parity wait on the stage's full barrier cannot
// match an earlier use of the same parity.
__device__ inline bool wait_armed(const WaitCtx &w, const int *armed, int seq)
{
    uint64_t t0 = 0;
    for (int it = 0;; ++it) {
        if (*(const volatile int *)armed == seq) return true;
        if (*w.abort) return false;
        if (it == 64) t0 = globaltimer_ns();
        if (it > 64 && (it & 15) == 0 && deadline_passed(t0, w.timeout_ns)) {
            raise_timeout(w);
            return false;
        }
    }
}

// Waits for the phase of `bar` with the given parity to complete.
__device__ inline bool wait_mbar_phase(const WaitCtx &w, uint64_t *bar, uint32_t parity)
{
    uint64_t t0 = 0;
    for (int it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*w.abort) return false;
        if (it == 64) t0 = globaltimer_ns();
        if (it > 64 && (it & 15) == 0 && deadline_passed(t0, w.timeout_ns)) {
            raise_timeout(w);
            return false;
        }
    }
}

}  // namespace hfq
