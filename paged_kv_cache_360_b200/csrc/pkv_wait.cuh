// pkv_wait.cuh -- bounded mbarrier waits with a shared abort word, for the
// warp-specialised tensor-core kernels (prefill, shared-prefix decode).
//
// Every wait gives up after kWaitCycles SM cycles (about half a second): a
// protocol fault then costs each CTA a bounded delay, never a hang.  A wait
// that gives up raises the CTA's abort word, so that the other roles stop
// waiting too, and records PKV_DEVERR_WAIT_TIMEOUT in the caller's flag.
#pragma once

#include <stdint.h>

#include "pkv.h"
#include "pkv_ptx.cuh"

namespace pkv {

__device__ __forceinline__ void raise_flag(int32_t* err, int bit) {
    if (err) atomicOr(err, bit);
}

// Wait that also gives up when another role raised the abort word.
// Warp-uniform: every lane of the calling warp must call it.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity,
                                          volatile uint32_t* abort_word, int32_t* err) {
    bool ok = false;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_test(bar, parity)) {
            ok = true;
            break;
        }
        if (*abort_word || clock64() - t0 > kWaitCycles) break;
    }
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && *abort_word == 0u) {
        *abort_word = 1u;
        if ((threadIdx.x & 31) == 0) raise_flag(err, PKV_DEVERR_WAIT_TIMEOUT);
    }
    return ok;
}

// Single-thread variant (an MMA issuer).
__device__ __forceinline__ bool one_wait(uint32_t bar, uint32_t parity,
                                         volatile uint32_t* abort_word, int32_t* err) {
    const long long t0 = clock64();
    for (;;) {
        if (mbar_test(bar, parity)) return true;
        if (*abort_word) return false;
        if (clock64() - t0 > kWaitCycles) break;
    }
    *abort_word = 1u;
    raise_flag(err, PKV_DEVERR_WAIT_TIMEOUT);
    return false;
}

// Wait for completion, ignoring the abort word (draining copies and MMAs).
__device__ __forceinline__ void quiet_wait(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_test(bar, parity) && clock64() - t0 <= kWaitCycles) {
    }
}

}  // namespace pkv
