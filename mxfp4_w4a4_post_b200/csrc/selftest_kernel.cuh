// Self-test of the bounded device waits the GEMM kernel relies on (failure detection;
// the pages have no counterpart).
//
// Two CTAs, 96 threads each, run the GEMM's own wait routines against waits that
// cannot succeed, with a short limit, and record what happened:
//   CTA 0, warp 0: wait_or_abort on an mbarrier nothing arrives at, limit limit_ns;
//                  gives up, records kErrTimeoutProducer, raises the CTA abort flag.
//   CTA 0, warp 1: the same kind of wait with the normal limit; must leave as soon as
//                  it sees the abort flag, without recording a code of its own.
//   CTA 0, warp 2: waits on a barrier it completes itself; must succeed.
//   CTA 1, warps 0-2: the exit agreement of the kernel's warp groups (bar_and, the
//                  named barrier that returns whether a condition held in every warp):
//                  warp 0 waits on an mbarrier nothing arrives at, limit limit_ns, and
//                  gives up (kErrTimeoutSet); warps 1 and 2 wait on barriers that
//                  complete; all three must then agree to leave, and none is held.
// Nothing else is in flight (no TMA, no tensor memory), so a kernel that gives up
// simply returns and the context stays usable.
#pragma once

#include <cstdint>

#include "gemm_kernel.cuh"

namespace macaq {

constexpr int kSelftestWords = 10;

// out[0..2]  CTA 0 warps 0, 1, 2: wait result (1 = completed, 0 = gave up)
// out[3]     CTA 0 error word after all warps returned
// out[4..5]  CTA 0 warps 0, 1: time spent in the wait, ns
// out[6]     CTA 1: the agreed result seen by warp 1 (1 = all waits completed)
// out[7]     CTA 1 error word
// out[8]     CTA 1 warp 0: time spent in its wait, ns
// out[9]     CTA 1 warp 2: its own wait result
__global__ void __launch_bounds__(96, 1) wait_selftest_kernel(uint64_t limit_ns, long long* out) {
    __shared__ __align__(8) uint64_t bars[3];
    __shared__ int abort_flag;
    __shared__ int err;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 3; ++i) ptx::mbar_init(&bars[i], 1);
        ptx::fence_mbar_init();
        abort_flag = 0;
        err = 0;
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        if (warp == 2 && lane == 0) ptx::mbar_arrive(&bars[2]);
        const uint64_t t0 = global_timer_ns();
        bool ok;
        if (warp == 0)
            ok = warp_wait(&bars[0], 0, &abort_flag, &err, kErrTimeoutProducer, limit_ns);
        else if (warp == 1)
            ok = warp_wait(&bars[1], 0, &abort_flag, &err, kErrTimeoutEpilogue);
        else
            ok = warp_wait(&bars[2], 0, &abort_flag, &err, kErrTimeoutMma);
        const uint64_t dt = global_timer_ns() - t0;
        if (lane == 0) {
            out[warp] = ok ? 1 : 0;
            if (warp < 2) out[4 + warp] = (long long)dt;
        }
        __syncthreads();
        if (threadIdx.x == 0) out[3] = err;
    } else {
        // warps 1 and 2 complete their own barriers; warp 0's never completes
        if (warp >= 1 && lane == 0) ptx::mbar_arrive(&bars[warp]);
        const uint64_t t0 = global_timer_ns();
        const bool own = warp_wait(&bars[warp], 0, &abort_flag, &err, warp == 0 ? kErrTimeoutSet : kErrTimeoutMma,
                                   warp == 0 ? limit_ns : kWaitLimitNs);
        const uint64_t dt = global_timer_ns() - t0;
        const bool agreed = bar_and(5, 96, own);
        if (lane == 0 && warp == 0) out[8] = (long long)dt;
        if (lane == 0 && warp == 1) out[6] = agreed ? 1 : 0;
        if (lane == 0 && warp == 2) out[9] = own ? 1 : 0;
        __syncthreads();
        if (threadIdx.x == 0) out[7] = err;
    }
}

}  // namespace macaq
