// fa_common.cuh -- device error word and time-bounded waits shared by the kernels.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"

namespace fa {

// Bits of the device error word (read and cleared by fa_get_error).
enum : unsigned int {
    kErrTimeout = 1u,      // a pipeline wait exceeded its limit
    kErrSeqlenRange = 2u,  // a decode length was outside [0, Nmax] and was clamped
    kErrPageRange = 4u,    // a block-table entry was outside [0, num_pages); its keys read as 0
    kErrDebugBounds = 8u,  // debug builds: an address computed by a kernel failed its bounds check
};

// One word per process, in the library's own device memory.
__device__ unsigned int g_error_word = 0;

__device__ __forceinline__ void raise_error(unsigned int bit) { atomicOr(&g_error_word, bit); }

// Debug builds (compiled with FA_DEBUG_CHECKS): every global-memory index that a kernel
// computes by hand (outputs, partials, scales, block-table and q rows) is checked against
// the size of its buffer before the access; a failed check records kErrDebugBounds and the
// access is skipped, so a bad index is reported instead of touching memory outside the
// buffer.  (TMA copies are bounds-checked by the copy engine itself.)  In release builds the
// check is the constant true and costs nothing.
#ifdef FA_DEBUG_CHECKS
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

__device__ __forceinline__ bool in_bounds(long long idx, long long n)
{
    if (!kDebugChecks) return true;
    if (idx >= 0 && idx < n) return true;
    raise_error(kErrDebugBounds);
    return false;
}

// Per-CTA stop flag (in shared memory): set by the first role whose wait runs out, read
// by every other role at each wait so that the whole CTA winds down together.
struct StopFlag {
    volatile int *flag;
    uint64_t limit_ns;

    __device__ __forceinline__ bool stopped() const { return *flag != 0; }
    __device__ __forceinline__ void stop() const { *flag = 1; }
};

// Wait, by all 32 lanes of a warp together, for the phase of `bar` with parity `parity`.
// Returns false if the CTA was told to stop or the limit ran out (which records
// kErrTimeout and tells the CTA to stop).  The outcome is warp-uniform, so that
// warp-collective tensor-memory instructions after it stay converged.
__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, const StopFlag &sf)
{
    if (__all_sync(0xffffffffu, ptx::mbar_test(bar, parity))) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (__all_sync(0xffffffffu, ptx::mbar_test(bar, parity))) return true;
        if ((n & 31u) == 0u) {
            int give_up = 0;
            if ((threadIdx.x & 31u) == 0u) {
                if (sf.stopped()) {
                    give_up = 1;
                } else if (ptx::globaltimer_ns() - t0 > sf.limit_ns) {
                    raise_error(kErrTimeout);
                    sf.stop();
                    give_up = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
        }
    }
}

// A barrier among the warps of a role built on an mbarrier (initialised with a count of
// one arrival per warp), so that -- unlike bar.sync -- waiting on it is time-bounded and
// honours the CTA stop flag.  Every participating warp calls sync() the same number of
// times; each call is one phase.
struct GroupBarrier {
    uint64_t *bar;
    uint32_t phase;

    __device__ __forceinline__ bool sync(const StopFlag &sf)
    {
        __syncwarp();
        if ((threadIdx.x & 31u) == 0u) ptx::mbar_arrive(bar);
        const bool ok = wait_warp(bar, phase, sf);
        phase ^= 1u;
        return ok;
    }
};

}  // namespace fa
