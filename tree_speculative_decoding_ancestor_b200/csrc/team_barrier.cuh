// Exchange of one partial result per CTA among the CTAs of one team of a
// cooperative launch, with a bounded wait (used by the stochastic walk; the
// wait probe exercises the same code).
#pragma once

#include <stdint.h>

namespace tsd {

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void st_release(int *p, int v)
{
    asm volatile("st.release.gpu.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Exchange number n of a team of K CTAs (n = 1, 2, ... counts the team's
// exchanges; every CTA of the team makes the same ones).  Thread 0 of CTA k
// has written slots[k] (this exchange's buffer) and now publishes it: a
// release store of n into tags[k].  Lanes 0 .. K-1 of warp 0 each wait for
// tags[lane] == n (acquire) and then load slots[lane] into `val`.  So the
// arrival and the read of the partials are one round trip, with no shared
// counter.  A wait gives up after `limit_ns`, or once the team's abort flag
// is set, and then raises the flag itself, which releases the other CTAs.
// Called by every thread of the CTA; false after an abort (every thread).
// Buffers alternate by exchange parity: a CTA writes a buffer again only
// after exchange n + 1, which every CTA enters after reading exchange n.
__device__ __forceinline__ bool team_exchange(const double2 *slots, int *tags, int k, int K,
                                              int n, int *abort, double2 &val, int *sh_ok,
                                              unsigned long long limit_ns)
{
    __syncthreads();
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0)
        st_release(tags + k, n);
    if (threadIdx.x < 32) {
        bool ok = true;
        if (lane < K) {
            const unsigned long long t0 = global_ns();
            for (unsigned it = 0;; ++it) {
                if (ld_acquire(tags + lane) == n)
                    break;
                if (*(volatile int *)abort) {
                    ok = false;
                    break;
                }
                if ((it & 15u) == 15u && global_ns() - t0 > limit_ns) {
                    atomicExch(abort, 1);
                    ok = false;
                    break;
                }
                __nanosleep(32);
            }
            if (ok)
                val = __ldcg(slots + lane);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (lane == 0)
            *sh_ok = ok ? 1 : 0;
    }
    __syncthreads();
    return *sh_ok != 0;
}

}  // namespace tsd
