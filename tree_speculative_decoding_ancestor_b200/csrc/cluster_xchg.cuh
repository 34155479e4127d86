// Exchange of one double2 per CTA among the CTAs of a thread-block cluster,
// through distributed shared memory, with a bounded wait (used by the
// stochastic walk; the wait probe exercises the same code).
//
// Every CTA holds xslot[2][kXchgMax] and two mbarriers xbar[2] (count = the
// cluster size K).  Exchange n uses buffer n & 1: thread t < K of CTA k stores
// the CTA's value into slot [n & 1][k] of CTA t and arrives on CTA t's
// xbar[n & 1] (release at cluster scope); then every thread of every CTA
// waits on its own xbar[n & 1] for phase n >> 1 (acquire at cluster scope)
// and reads the K values from its own shared memory.  Buffer n & 1 is written
// again only at exchange n + 2, which no CTA reaches before every CTA has
// arrived at exchange n + 1 -- after it read the values of exchange n.
#pragma once

#include <stdint.h>

namespace tsd {

constexpr int kXchgMax = 16;   // CTAs per cluster at most

struct XchgShared {
    double2 slot[2][kXchgMax];
    unsigned long long bar[2];
};

__device__ __forceinline__ uint32_t xchg_smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// The address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Every thread of every CTA of the cluster (hardware barrier; all CTAs reach
// it on every path: at the start, after the barriers are initialised, and
// before exit, so that no CTA leaves while a peer may still write to it).
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release;\n\t"
                 "barrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ unsigned long long xchg_global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Thread 0 sets up the barriers; the caller then runs cluster_sync_all().
__device__ __forceinline__ void xchg_init(XchgShared *x, int K)
{
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(xchg_smem_addr(&x->bar[i])),
                         "r"(K)
                         : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
}

// Exchange n (counted from 0 by the caller, the same sequence in every CTA):
// `v` is this CTA's value (needed on threads 0 .. K-1).  Returns false on
// every thread of the CTA when the wait ran past limit_ns; true once the K
// values are in x->slot[n & 1].  Ends with a CTA barrier.
__device__ __forceinline__ bool cluster_exchange(XchgShared *x, int K, int n, double2 v,
                                                 unsigned long long limit_ns)
{
    const int buf = n & 1;
    const uint32_t parity = (uint32_t)(n >> 1) & 1u;
    if ((int)threadIdx.x < K) {
        const uint32_t rank = cluster_ctarank();
        const uint32_t dst = cluster_map(xchg_smem_addr(&x->slot[buf][rank]), threadIdx.x);
        const uint32_t bar = cluster_map(xchg_smem_addr(&x->bar[buf]), threadIdx.x);
        asm volatile("st.shared::cluster.v2.f64 [%0], {%1, %2};" ::"r"(dst), "d"(v.x), "d"(v.y)
                     : "memory");
        asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar)
                     : "memory");
    }
    const uint32_t mine = xchg_smem_addr(&x->bar[buf]);
    int ok = 1;
    unsigned long long t0 = 0;
    for (uint32_t it = 0;; ++it) {
        uint32_t done;
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(done)
                     : "r"(mine), "r"(parity)
                     : "memory");
        if (done)
            break;
        if (it == 0)
            t0 = xchg_global_ns();
        else if ((it & 15u) == 0u && xchg_global_ns() - t0 > limit_ns) {
            ok = 0;
            break;
        }
    }
    return __syncthreads_and(ok) != 0;
}

}  // namespace tsd
