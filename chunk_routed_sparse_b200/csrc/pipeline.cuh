// Bounded mbarrier waits shared by the warp-specialised kernels.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace moc {

constexpr uint64_t kTimeoutNs = 2000000000ull;  // every device-side wait gives up after 2 s

// Wait for the phase of `parity` to complete. Returns false on timeout (after
// recording ERR_TIMEOUT and the site code `where` in the workspace header and
// raising the CTA's abort flag) or when another role already aborted.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort,
                                         int32_t* hdr, int where) {
    using namespace sm100;
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 0) {
            if (*abort) return false;
            if (globaltimer() - t0 > kTimeoutNs) {
                set_error(hdr, ERR_TIMEOUT, where);
                *abort = 1;
                return false;
            }
        }
    }
}

// The same wait, made uniform across the warp (warps that execute
// warp-collective tcgen05.ld/st right after it).
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, volatile int* abort,
                                              int32_t* hdr, int where) {
    const bool ok = wait_bar(bar, parity, abort, hdr, where);
    return __all_sync(0xffffffffu, ok);
}

// Bounded drain wait that ignores the abort flag (used before releasing
// resources: outstanding copies or MMAs must land first).
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity, int32_t* hdr, int where) {
    using namespace sm100;
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kTimeoutNs) {
            set_error(hdr, ERR_TIMEOUT, where);
            return;
        }
    }
}

}  // namespace moc
