// Barrier over the CTAs of one team of a cooperative launch, with a bounded
// wait (used by the stochastic walk; the wait probe exercises the same code).
#pragma once

#include <stdint.h>

namespace tsd {

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// `team` = {arrivals, abort}; `target` = the team's CTA count x the number of
// barriers the team has entered, this one included.  Thread 0 publishes the
// CTA's earlier global writes (a release-ordered arrival) and spins on the
// counter; after `limit_ns` it raises the team's abort flag, which releases
// the other CTAs as well.  False after an abort (every thread of the CTA).
__device__ __forceinline__ bool team_barrier(int2 *team, int target, int *sh_ok,
                                             unsigned long long limit_ns)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        int *arrive = &team->x;
        volatile int *abort = &team->y;
        asm volatile("red.release.gpu.add.s32 [%0], 1;" ::"l"(arrive) : "memory");
        const unsigned long long t0 = global_ns();
        int ok = 1;
        for (;;) {
            int v;
            asm volatile("ld.acquire.gpu.b32 %0, [%1];" : "=r"(v) : "l"(arrive) : "memory");
            if (v >= target)
                break;
            if (*abort) {
                ok = 0;
                break;
            }
            if (global_ns() - t0 > limit_ns) {
                atomicExch(&team->y, 1);
                ok = 0;
                break;
            }
            __nanosleep(64);
        }
        *sh_ok = ok;
    }
    __syncthreads();
    return *sh_ok != 0;
}

}  // namespace tsd
