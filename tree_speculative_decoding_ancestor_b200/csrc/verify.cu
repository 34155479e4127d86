// Tree verification from the target model's logits (SpecInfer explainer,
// section "ツリー検証アルゴリズム").
//
// greedy (a node is matched when its token is the argmax of its parent's row;
// the result is the deepest node whose whole root path is matched, lowest
// index on ties, and the argmax of that node's row as the bonus token)
//   greedy_walk_kernel      (batches whose logits exceed 64 MiB) one CTA per
//                           sequence walks the matched nodes level by level
//                           from the root, taking the argmax of each visited
//                           row: it reads the root row and the rows of
//                           matched nodes only;
//   greedy_rows_kernel      (smaller batches) one CTA per logits row whose
//                           node has children: argmax (lowest index on ties),
//                           float4 loads, several in flight per thread;
//   greedy_finalize_kernel  one CTA per sequence after it: the nodes whose
//                           whole root path matches, the deepest, and the
//                           argmax of its row (computed here for a leaf).
// stochastic (multi-step speculative sampling)
//   mss_walk_kernel         one launch.  Each sequence is walked by a team of
//                           K CTAs, CTA k owning one contiguous chunk of the
//                           vocabulary.  At the current node's row the team
//                           computes m = max l and Z = sum exp((l-m)/T) in
//                           fp64, then tries the children in ascending index:
//                           child c with token x is accepted iff p(x) > 0 and
//                           u_c * q_c(x) <= p(x) (fp64, CUDA's exp, every
//                           CTA taking the same decision from the same
//                           numbers); after a rejection the team sums
//                           S = sum max(0, p - q_c) and p becomes
//                           max(0, p - q_c) / S.  An accepted child's row is
//                           next.  Every pass also leaves the current
//                           distribution's sum over each chunk (z_k/Z, or
//                           S_k/S after a rejection); where the walk stops,
//                           the chunk whose running sum passes u_sample[row]
//                           is scanned (fp64 block scan) by its CTA for the
//                           token -- the draw costs no exchange.
//                           Only rows on the accepted path are read.  A team
//                           is a thread-block cluster exchanging its partials
//                           through distributed shared memory (vocabularies
//                           up to 8 x 4096 entries) or K CTAs of a cooperative
//                           launch exchanging them through workspace slots
//                           and a per-team arrival counter; every wait is
//                           bounded (TSD_DEV_TIMEOUT).
//
// Cached form (chunks of at most 4096 entries): each CTA keeps its chunk of
// the current distribution in shared memory in fp64, scaled (p = pc * g), so
// a rejected sibling costs one pass over its q chunk and an in-place
// renormalisation; with 16-byte aligned rows the chunks a pass reads arrive
// in shared memory by bulk copies issued one pass ahead.  Otherwise p^(n)(x)
// is recomputed per element from the logits row, the rejected siblings' q
// rows and their normalisers.  The bulk sums (Z, S, the CDF) use a
// table-driven fp64 exp and reciprocals; the acceptance tests use CUDA's fp64
// exp and the reciprocals of T, Z and the S_j.  Both agree with a sequential
// fp64 evaluation of the formulas to ~1e-15 relative, so a decision can only
// differ when its uniform lies within that distance of the boundary.
#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdlib>
#include <cstring>

#include "cluster_xchg.cuh"
#include "fp64_exp.cuh"
#include "sm100_ptx.cuh"
#include "team_barrier.cuh"
#include "tsd_common.cuh"

namespace tsd {

namespace {

constexpr int kRowThreads = 512;
constexpr int kFinThreads = 1024;
constexpr int kWalkThreads = 256;
constexpr int kWalkWarps = kWalkThreads / 32;
constexpr int kTeamMax = 32;          // CTAs per team: one partial per lane of a warp
constexpr int kTeamMinChunk = 2048;   // vocabulary entries per CTA, at least
constexpr int kClusterTeam = 8;       // CTAs per cluster team at most (portable cluster size)
constexpr int kWalkMaxCtas = 1024;    // grid cap (sets the workspace slots)
constexpr unsigned long long kTeamWaitNs = 2000000000ull;   // bound of one barrier wait
constexpr int kCacheGroups = 4;       // groups of 4 entries per thread in the cached walk
constexpr int kCacheChunk = 4 * kCacheGroups * kWalkThreads;   // 4096 entries: 32 KB fp64
constexpr int kStageBytes = 2 * 2 * kCacheChunk * 4;   // staged chunks: 2 sets x (logits, q)
constexpr int kDecCache = 8;          // children per row whose test operands are prefetched
constexpr int kDecOps = 2 * kDecCache + kDecCache * (kDecCache + 1) / 2;   // 52 loads
static_assert(4 * kDecOps <= kWalkThreads, "one acceptance operand per fourth thread");

struct VerifyWs {
    double2 *slot;     // [2][kWalkMaxCtas]  per-CTA partials, by barrier parity
    int2 *team;        // [kWalkMaxCtas]     {arrivals, abort} per team, zeroed per call
    int32_t *argmax;   // [B][Tmax+1]        greedy: argmax of rows with children
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Fixed part first: the stochastic call uses only that.
constexpr size_t kWalkBytes = ((2 * kWalkMaxCtas * sizeof(double2) + 255) & ~(size_t)255) +
                              ((kWalkMaxCtas * sizeof(int2) + 255) & ~(size_t)255);

VerifyWs carve(void *ws)
{
    char *p = static_cast<char *>(ws);
    VerifyWs w;
    w.slot = reinterpret_cast<double2 *>(p);
    p += align256(2 * kWalkMaxCtas * sizeof(double2));
    w.team = reinterpret_cast<int2 *>(p);
    p += align256(kWalkMaxCtas * sizeof(int2));
    w.argmax = reinterpret_cast<int32_t *>(p);
    return w;
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ bool better(float v, int i, float bv, int bi)
{
    return v > bv || (v == bv && i < bi);
}

template <int NT>
__device__ void block_argmax(float &v, int &i, float *shv, int *shi)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (better(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
    if (lane == 0) {
        shv[warp] = v;
        shi[warp] = i;
    }
    __syncthreads();
    if (warp == 0) {
        v = lane < NW ? shv[lane] : -INFINITY;
        i = lane < NW ? shi[lane] : INT_MAX;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, v, o);
            const int oi = __shfl_xor_sync(0xffffffffu, i, o);
            if (better(ov, oi, v, i)) {
                v = ov;
                i = oi;
            }
        }
        if (lane == 0) {
            shv[0] = v;
            shi[0] = i;
        }
    }
    __syncthreads();
    v = shv[0];
    i = shi[0];
    __syncthreads();
}

template <int NT>
__device__ float block_max(float v, float *sh)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_max(v);
    if (lane == 0)
        sh[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < NW ? sh[lane] : -INFINITY;
        v = warp_max(v);
        if (lane == 0)
            sh[0] = v;
    }
    __syncthreads();
    v = sh[0];
    __syncthreads();
    return v;
}

// Block reductions for the walk: warp partials through shared memory, then
// every thread combines them itself in warp order (the same value on every
// thread, and two barriers instead of three).
template <int NT>
__device__ double block_sum(double v, double *sh)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    if (lane == 0)
        sh[warp] = v;
    __syncthreads();
    v = 0.0;
#pragma unroll
    for (int w = 0; w < NW; ++w)
        v += sh[w];
    __syncthreads();
    return v;
}

template <int NT>
__device__ int block_min_int(int v, int *sh)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0)
        sh[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < NW ? sh[lane] : INT_MAX;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0)
            sh[0] = v;
    }
    __syncthreads();
    v = sh[0];
    __syncthreads();
    return v;
}

template <int NT>
__device__ int block_max_int(int v, int *sh)
{
    return -block_min_int<NT>(-v, sh);
}

// The CTA's largest m and largest index last in one block reduction.
template <int NT>
__device__ void block_max_last(float &m, int &last, float *shf, int *shi)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    auto warp_reduce = [&]() {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
        }
    };
    warp_reduce();
    if (lane == 0) {
        shf[warp] = m;
        shi[warp] = last;
    }
    __syncthreads();
    m = -INFINITY;
    last = -1;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        m = fmaxf(m, shf[w]);
        last = max(last, shi[w]);
    }
    __syncthreads();
}

// The CTA's (sum s, largest index last) in one block reduction.
template <int NT>
__device__ void block_sum_last(double &s, int &last, double *shd, int *shi)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    auto warp_reduce = [&]() {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s += __shfl_xor_sync(0xffffffffu, s, o);
            last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
        }
    };
    warp_reduce();
    if (lane == 0) {
        shd[warp] = s;
        shi[warp] = last;
    }
    __syncthreads();
    s = 0.0;
    last = -1;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        s += shd[w];
        last = max(last, shi[w]);
    }
    __syncthreads();
}

// Row argmax (lowest index among the maxima).  Each thread keeps NB float4
// loads in flight per batch, the last batch predicated (no tail of single
// loads).  NB = 8 (a 32000-entry row in one batch for 1024 threads) where a
// row's latency is the cost: the greedy walk and finalize; NB = 4 where many
// CTAs per SM keep the bytes in flight: the all-rows scan, whose occupancy
// the extra registers would cut.
template <int NT, int NB = 8>
__device__ int row_argmax(const float *__restrict__ row, int V, float *shv, int *shi)
{
    float bv = -INFINITY;
    int bi = INT_MAX;
    if ((V & 3) == 0) {
        const float4 *r4 = reinterpret_cast<const float4 *>(row);
        const int n4 = V >> 2;
        for (int j0 = threadIdx.x; j0 < n4; j0 += NB * NT) {
            float4 x[NB];
#pragma unroll
            for (int k = 0; k < NB; ++k)
                if (j0 + k * NT < n4)
                    x[k] = __ldg(r4 + j0 + k * NT);
#pragma unroll
            for (int k = 0; k < NB; ++k) {
                if (j0 + k * NT >= n4)
                    break;
                const int i0 = 4 * (j0 + k * NT);
                if (better(x[k].x, i0, bv, bi)) { bv = x[k].x; bi = i0; }
                if (better(x[k].y, i0 + 1, bv, bi)) { bv = x[k].y; bi = i0 + 1; }
                if (better(x[k].z, i0 + 2, bv, bi)) { bv = x[k].z; bi = i0 + 2; }
                if (better(x[k].w, i0 + 3, bv, bi)) { bv = x[k].w; bi = i0 + 3; }
            }
        }
    } else {
        for (int j = threadIdx.x; j < V; j += NT) {
            const float x = __ldg(row + j);
            if (better(x, j, bv, bi)) { bv = x; bi = j; }
        }
    }
    block_argmax<NT>(bv, bi, shv, shi);
    return bi == INT_MAX ? 0 : bi;
}

// Asynchronous 4- and 8-byte copies from global to shared memory (aligned to
// their size), and the wait for all of this thread's copies.
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async8(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Starts an L2 prefetch of bytes [p, p + bytes) (p 16-byte aligned, bytes a
// multiple of 16): one bulk request, nothing waits for it.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Per-row state of multi-step speculative sampling.
struct RowState {
    double m, inv_temp, temp, Z, inv_Z;
    int n;                         // siblings rejected so far (-1: malformed input)
    const float *q[kMaxTree];      // their SSM rows
    double S[kMaxTree];            // their residual normalisers
    double inv_S[kMaxTree];        // 1/S (0 when S == 0: p unchanged)
};

// Four consecutive fp32 values starting at x0 (0 beyond V); one float4 load
// when the row is 16-byte aligned and V % 4 == 0 (VEC).
template <bool VEC>
__device__ __forceinline__ void load4(const float *__restrict__ p, int x0, int V, float (&v)[4])
{
    if (VEC) {
        if (x0 < V) {
            const float4 t = __ldg(reinterpret_cast<const float4 *>(p + x0));
            v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
        } else {
            v[0] = v[1] = v[2] = v[3] = 0.f;
        }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            v[k] = x0 + k < V ? __ldg(p + x0 + k) : 0.f;
    }
}

// Four values of a chunk [x_lo, ..) starting at x0 < x_hi: from the global
// row (SMEM false: p is the row) or from the chunk staged in shared memory
// (SMEM: p is the chunk's first entry, 16-byte aligned).
template <bool VEC, bool SMEM>
__device__ __forceinline__ void load4c(const float *p, int x0, int x_lo, int V, float (&v)[4])
{
    if (SMEM) {
        const float4 t = *reinterpret_cast<const float4 *>(p + (x0 - x_lo));
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
        load4<VEC>(p, x0, V, v);
    }
}

// p^(n)(x) for x in [x0, x0+4) (0 beyond V) for the bulk sums (`table`
// unscaled: p^(0) = table_exp(..) / Z); the loads of each rejected sibling's
// row are issued together.
template <bool VEC>
__device__ __forceinline__ void p_bulk4(const float *__restrict__ row, int x0, int V,
                                        const RowState &st, const double *table, double (&p)[4])
{
    float l[4];
    load4<VEC>(row, x0, V, l);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        p[k] = x0 + k < V ? table_exp(((double)l[k] - st.m) * st.inv_temp, table) * st.inv_Z
                          : 0.0;
    for (int j = 0; j < st.n; ++j) {
        if (st.S[j] > 0.0) {
            float q[4];
            load4<VEC>(st.q[j], x0, V, q);
            const double is = st.inv_S[j];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const double r = p[k] - (double)q[k];
                p[k] = (r > 0.0 ? r : 0.0) * is;
            }
        }
    }
}

// One pass over the CTA's chunk [x_lo, x_hi) of a logits row: the chunk's
// max m_k, z_k = sum exp((l - m_k)/T) and (in *last) the largest x with a
// finite logit, -1 if none.  Each thread keeps a running max and rescales
// its sum when the max rises.
template <bool VEC>
__device__ double2 chunk_max_z(const float *__restrict__ row, int x_lo, int x_hi, int V,
                               double inv_temp, const double *table, float *shf, double *shd,
                               int *shi, int *last_out)
{
    float mt = -INFINITY;
    double zt = 0.0;
    int last = -1;
    auto group = [&](const float (&l)[4], int x0) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (l[k] > -INFINITY)
                last = x0 + k;
        const float m4 = fmaxf(fmaxf(l[0], l[1]), fmaxf(l[2], l[3]));
        if (m4 > mt) {
            if (mt != -INFINITY)
                zt *= table_exp(((double)mt - (double)m4) * inv_temp, table);
            mt = m4;
        }
        if (mt != -INFINITY) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                zt += table_exp(((double)l[k] - (double)mt) * inv_temp, table);
        }
    };
    for (int x0 = x_lo + 4 * threadIdx.x; x0 < x_hi; x0 += 8 * kWalkThreads) {
        const int x1 = x0 + 4 * kWalkThreads;
        float l0[4], l1[4];
        load4<VEC>(row, x0, V, l0);
        load4<VEC>(row, x1, V, l1);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (x0 + k >= x_hi)
                l0[k] = -INFINITY;
            if (x1 + k >= x_hi)
                l1[k] = -INFINITY;
        }
        group(l0, x0);
        group(l1, x1);
    }
    // the chunk's max and last in one reduction, then each thread rescales
    // its own sum to the chunk max (in parallel), then one sum
    float mk = mt;
    block_max_last<kWalkThreads>(mk, last, shf, shi);
    *last_out = last;
    const double zs =
        mt == -INFINITY ? 0.0 : zt * table_exp(((double)mt - (double)mk) * inv_temp, table);
    return make_double2((double)mk, block_sum<kWalkThreads>(zs, shd));
}

// Over the CTA's chunk: sum max(0, p^(n)(x) - q(x)) and (in *last) the
// largest x where that is positive (-1 if none).  x_lo is a multiple of 4
// and x_hi is one or V, so the groups of four never straddle x_hi inside the
// vocabulary.
template <bool VEC>
__device__ double chunk_residual(const float *__restrict__ row, const float *__restrict__ q,
                                 int x_lo, int x_hi, int V, const RowState &st,
                                 const double *table, double *shd, int *shi, int *last_out)
{
    double s = 0.0;
    int last = -1;
    for (int x0 = x_lo + 4 * threadIdx.x; x0 < x_hi; x0 += 8 * kWalkThreads) {
        const int x1 = x0 + 4 * kWalkThreads;
        double p0[4], p1[4] = {0.0, 0.0, 0.0, 0.0};
        float q0[4], q1[4];
        p_bulk4<VEC>(row, x0, V, st, table, p0);
        if (x1 < x_hi)
            p_bulk4<VEC>(row, x1, V, st, table, p1);
        load4<VEC>(q, x0, V, q0);
        load4<VEC>(q, x1 < x_hi ? x1 : V, V, q1);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const double d0 = p0[k] - (double)q0[k], d1 = p1[k] - (double)q1[k];
            s += (d0 > 0.0 ? d0 : 0.0) + (d1 > 0.0 ? d1 : 0.0);
            if (d0 > 0.0)
                last = max(last, x0 + k);
            if (d1 > 0.0)
                last = max(last, x1 + k);
        }
    }
    block_sum_last<kWalkThreads>(s, last, shd, shi);
    *last_out = last;
    return s;
}

// ---- the cached form: a CTA keeps its chunk of the current distribution in
// shared memory (kCacheChunk entries at most), scaled: p(x) = pc[x - x_lo] * g.
// Thread tid owns the groups of four entries tid, tid + 256, tid + 512 and
// tid + 768 of the chunk in every pass, so each pass reads the global rows
// once with coalesced loads and the cached values need no barrier between the
// passes of a row.

// m/Z pass: the chunk's logits -> registers, the chunk max m_k (and the
// largest x with a finite logit), then pc = exp((l - m_k)/T) and its sum.
template <bool VEC, bool SMEM>
__device__ double2 chunk_max_z_cached(const float *__restrict__ row, int x_lo, int x_hi, int V,
                                      double inv_temp, const double *table, double *pc,
                                      float *shf, double *shd, int *shi, int *last_out)
{
    float l[4 * kCacheGroups];
    float mt = -INFINITY;
    int last = -1;
#pragma unroll
    for (int m = 0; m < kCacheGroups; ++m) {
        const int x0 = x_lo + 4 * (threadIdx.x + kWalkThreads * m);
        float v[4];
        if (x0 < x_hi)
            load4c<VEC, SMEM>(row, x0, x_lo, V, v);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float lv = (x0 + k < x_hi) ? v[k] : -INFINITY;
            l[4 * m + k] = lv;
            mt = fmaxf(mt, lv);
            if (lv > -INFINITY)
                last = x0 + k;
        }
    }
    block_max_last<kWalkThreads>(mt, last, shf, shi);
    *last_out = last;
    // no branches here, so that the 16 exponentials of a thread interleave:
    // entries past x_hi hold -inf (their pc entries, 0, are never read) and
    // -inf goes to 0 (also when the whole chunk is -inf)
    const double md = (double)mt;
    double e[4 * kCacheGroups];
#pragma unroll
    for (int i = 0; i < 4 * kCacheGroups; ++i) {
        const double x = ((double)l[i] - md) * inv_temp;
        e[i] = table_exp(l[i] == -INFINITY ? -INFINITY : x, table);
    }
    double z = 0.0;
#pragma unroll
    for (int m = 0; m < kCacheGroups; ++m) {
        const int i0 = 4 * (threadIdx.x + kWalkThreads * m);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            pc[i0 + k] = e[4 * m + k];
            z += e[4 * m + k];
        }
    }
    return make_double2((double)mt, mt == -INFINITY ? 0.0 : block_sum<kWalkThreads>(z, shd));
}

// Residual pass: S_k = sum over the chunk of max(0, p(x) - q(x)) with p(x) =
// pc * g, and the largest x where that is positive.
template <bool VEC, bool SMEM>
__device__ double chunk_residual_cached(const float *__restrict__ q, int x_lo, int x_hi, int V,
                                        const double *pc, double g, double *shd, int *shi,
                                        int *last_out)
{
    double s = 0.0;
    int last = -1;
#pragma unroll
    for (int m = 0; m < kCacheGroups; ++m) {
        const int i0 = 4 * (threadIdx.x + kWalkThreads * m);
        const int x0 = x_lo + i0;
        if (x0 >= x_hi)
            continue;
        float qv[4];
        load4c<VEC, SMEM>(q, x0, x_lo, V, qv);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (x0 + k < x_hi) {
                const double r = pc[i0 + k] * g - (double)qv[k];
                if (r > 0.0) {
                    s += r;
                    last = x0 + k;
                }
            }
        }
    }
    block_sum_last<kWalkThreads>(s, last, shd, shi);
    *last_out = last;
    return s;
}

// After a rejection with residual sum S > 0: pc = max(0, pc * g - q) / S (the
// q chunk comes from L1, just read), so that g becomes 1.  Each thread
// rewrites only the entries it owns.
template <bool VEC, bool SMEM>
__device__ void chunk_renormalise_cached(const float *__restrict__ q, int x_lo, int x_hi, int V,
                                         double *pc, double g, double inv_S)
{
#pragma unroll
    for (int m = 0; m < kCacheGroups; ++m) {
        const int i0 = 4 * (threadIdx.x + kWalkThreads * m);
        const int x0 = x_lo + i0;
        if (x0 >= x_hi)
            continue;
        float qv[4];
        load4c<VEC, SMEM>(q, x0, x_lo, V, qv);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (x0 + k < x_hi) {
                const double r = pc[i0 + k] * g - (double)qv[k];
                pc[i0 + k] = (r > 0.0 ? r : 0.0) * inv_S;
            }
        }
    }
}

// The draw inside the chunk, from the cached distribution: the smallest x
// with carry + sum_{x_lo <= y <= x} p(y) > u (fp64 block scan in order), or
// INT_MAX when rounding leaves the chunk's sum short of u.
__device__ int chunk_scan_cached(const double *pc, double g, int x_lo, int x_hi, double carry,
                                 double u, double *warp_tot, int *shi)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = x_lo; base < x_hi; base += 4 * kWalkThreads) {
        const int x0 = base + 4 * threadIdx.x;
        double p[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (x0 + k < x_hi)
                p[k] = pc[x0 + k - x_lo] * g;
        const double mine = ((p[0] + p[1]) + p[2]) + p[3];
        double incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += y;
        }
        if (lane == 31)
            warp_tot[warp] = incl;
        __syncthreads();
        double wbase = 0.0, tile = 0.0;
        for (int w2 = 0; w2 < kWalkWarps; ++w2) {
            const double t = warp_tot[w2];
            if (w2 < warp)
                wbase += t;
            tile += t;
        }
        double C = carry + wbase + (incl - mine);
        int found = INT_MAX;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            C += p[k];
            if (found == INT_MAX && x0 + k < x_hi && C > u)
                found = x0 + k;
        }
        found = block_min_int<kWalkThreads>(found, shi);   // ends with a barrier
        if (found != INT_MAX)
            return found;
        carry += tile;
    }
    return INT_MAX;
}

// The draw inside the chunk [x_lo, x_hi): the smallest x with
// carry + sum_{x_lo <= y <= x} p^(n)(y) > u (fp64 block scan in order), or
// INT_MAX when rounding leaves the chunk's sum short of u.
template <bool VEC>
__device__ int chunk_scan(const float *__restrict__ row, int x_lo, int x_hi, int V,
                          const RowState &st, const double *table, double carry, double u,
                          double *warp_tot, int *shi)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = x_lo; base < x_hi; base += 4 * kWalkThreads) {
        const int x0 = base + 4 * threadIdx.x;
        double p[4] = {0.0, 0.0, 0.0, 0.0};
        if (x0 < x_hi)
            p_bulk4<VEC>(row, x0, V, st, table, p);
        const double mine = ((p[0] + p[1]) + p[2]) + p[3];
        double incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += y;
        }
        if (lane == 31)
            warp_tot[warp] = incl;
        __syncthreads();
        double wbase = 0.0, tile = 0.0;
        for (int w2 = 0; w2 < kWalkWarps; ++w2) {
            const double t = warp_tot[w2];
            if (w2 < warp)
                wbase += t;
            tile += t;
        }
        double C = carry + wbase + (incl - mine);
        int found = INT_MAX;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            C += p[k];
            if (found == INT_MAX && x0 + k < x_hi && C > u)
                found = x0 + k;
        }
        found = block_min_int<kWalkThreads>(found, shi);   // ends with a barrier
        if (found != INT_MAX)
            return found;
        carry += tile;
    }
    return INT_MAX;
}

__device__ __forceinline__ bool sequence_ok(const int32_t *n_nodes, const int32_t *first_child,
                                            int b, int Tmax, int &T)
{
    T = n_nodes[b];
    return tree_header_ok(T, Tmax) && first_child[(size_t)b * (Tmax + 1)] != TSD_TREE_INVALID;
}

// ------------------------------------------------------------------ greedy
__global__ void __launch_bounds__(kRowThreads)
    greedy_rows_kernel(const float *__restrict__ logits, const int32_t *__restrict__ n_nodes,
                       const int32_t *__restrict__ first_child, int Tmax, int V,
                       int32_t *__restrict__ argmax_ws)
{
    __shared__ float shv[kRowThreads / 32];
    __shared__ int shi[kRowThreads / 32];
    const int r = blockIdx.x, b = blockIdx.y;
    int T;
    if (!sequence_ok(n_nodes, first_child, b, Tmax, T) || r > T)
        return;
    if (first_child[(size_t)b * (Tmax + 1) + r] < 0)
        return;   // leaf: its argmax is needed only if it ends the path
    const int a =
        row_argmax<kRowThreads, 4>(logits + ((size_t)b * (Tmax + 1) + r) * V, V, shv, shi);
    if (threadIdx.x == 0)
        argmax_ws[(size_t)b * (Tmax + 1) + r] = a;
}

__global__ void __launch_bounds__(kFinThreads)
    greedy_finalize_kernel(const float *__restrict__ logits, const int32_t *__restrict__ tokens,
                           const int32_t *__restrict__ parent,
                           const int32_t *__restrict__ n_nodes,
                           const uint32_t *__restrict__ mask,
                           const int32_t *__restrict__ first_child, int Tmax, int V,
                           const int32_t *__restrict__ argmax_ws, int32_t *__restrict__ out_tokens,
                           int32_t *__restrict__ out_path, int32_t *__restrict__ n_accepted,
                           int32_t *dev_status)
{
    constexpr int NW = kFinThreads / 32;
    __shared__ uint32_t matched[kMaskWords];
    __shared__ float shv[NW];
    __shared__ int shi[NW];
    const int b = blockIdx.x, u = threadIdx.x;
    const int W = (Tmax + 31) / 32;
    int T;
    if (!sequence_ok(n_nodes, first_child, b, Tmax, T)) {
        if (u == 0)
            n_accepted[b] = -1;
        return;
    }
    int tok = 0;
    bool bad = false;
    if (u < T) {
        tok = tokens[(size_t)b * Tmax + u];
        bad = tok < 0 || tok >= V;
    }
    if (u < kMaskWords)
        matched[u] = 0u;
    if (__syncthreads_or(bad)) {
        if (u == 0) {
            n_accepted[b] = -1;
            flag(dev_status, TSD_DEV_BAD_TOKEN);
        }
        return;
    }
    if (u < T) {
        const int p = parent[(size_t)b * Tmax + u];
        if (tok == argmax_ws[(size_t)b * (Tmax + 1) + p + 1])
            atomicOr(&matched[u >> 5], 1u << (u & 31));
    }
    __syncthreads();
    // Deepest node whose whole root path matched; ties -> smallest index.
    int key = -1;
    if (u < T) {
        bool full = true;
        int len = 0;
        for (int w = 0; w < W; ++w) {
            const uint32_t mw = mask[((size_t)b * Tmax + u) * W + w];
            full = full && (mw & ~matched[w]) == 0u;
            len += __popc(mw);
        }
        if (full)
            key = (len << 8) | (255 - u);
    }
    key = block_max_int<kFinThreads>(key, shi);
    const int t = key >= 0 ? 255 - (key & 255) : -1;
    const int n = key >= 0 ? key >> 8 : 0;
    if (t >= 0 && u < T) {
        const uint32_t *mt = mask + ((size_t)b * Tmax + t) * W;
        if ((mt[u >> 5] >> (u & 31)) & 1u) {
            int pos = 0;
            for (int w = 0; w < (u >> 5); ++w)
                pos += __popc(mt[w]);
            pos += __popc(mt[u >> 5] & ((1u << (u & 31)) - 1u));
            if (in_bounds(pos, Tmax, dev_status)) {
                out_path[(size_t)b * Tmax + pos] = u;
                out_tokens[(size_t)b * (Tmax + 1) + pos] = tok;
            }
        }
    }
    const int row = t + 1;
    int bonus;
    if (first_child[(size_t)b * (Tmax + 1) + row] >= 0)
        bonus = argmax_ws[(size_t)b * (Tmax + 1) + row];
    else
        bonus = row_argmax<kFinThreads>(logits + ((size_t)b * (Tmax + 1) + row) * V, V, shv,
                                        shi);
    if (u == 0 && in_bounds(n, Tmax + 1, dev_status)) {
        out_tokens[(size_t)b * (Tmax + 1) + n] = bonus;
        n_accepted[b] = n;
    }
}

// One CTA per sequence.  Level by level from the root, for each node of the
// level (the root, then the nodes whose whole root path matched, in the
// order they were collected) the block takes the argmax of the node's row
// and collects the children whose token equals it: the next level.  The last nonempty level
// holds the deepest fully matched nodes; its lowest index is the terminal,
// whose row argmax (already taken) is the bonus token.  The same answer as
// greedy_rows_kernel + greedy_finalize_kernel, from 1 + (matched nodes) rows.
__global__ void __launch_bounds__(kFinThreads)
    greedy_walk_kernel(const float *__restrict__ logits, const int32_t *__restrict__ tokens,
                       const int32_t *__restrict__ parent, const int32_t *__restrict__ n_nodes,
                       const int32_t *__restrict__ first_child, int Tmax, int V,
                       int32_t *__restrict__ out_tokens, int32_t *__restrict__ out_path,
                       int32_t *__restrict__ n_accepted, int32_t *dev_status)
{
    constexpr int NW = kFinThreads / 32;
    __shared__ float shv[NW];
    __shared__ int shi[NW];
    __shared__ int s_tok[kMaxTree], s_par[kMaxTree];
    __shared__ int s_level[2][kMaxTree + 1];   // nodes of the current / next level (-1 = root)
    __shared__ int s_count[2];
    const int b = blockIdx.x, u = threadIdx.x;
    int T;
    if (!sequence_ok(n_nodes, first_child, b, Tmax, T)) {
        if (u == 0)
            n_accepted[b] = -1;
        return;
    }
    bool bad = false;
    for (int i = u; i < T; i += kFinThreads) {
        const int tok = tokens[(size_t)b * Tmax + i];
        s_tok[i] = tok;
        s_par[i] = parent[(size_t)b * Tmax + i];   // validated by the mask build
        bad = bad || tok < 0 || tok >= V;
    }
    if (__syncthreads_or(bad)) {
        if (u == 0) {
            n_accepted[b] = -1;
            flag(dev_status, TSD_DEV_BAD_TOKEN);
        }
        return;
    }
    if (u == 0) {
        s_level[0][0] = -1;
        s_count[0] = 1;
    }
    __syncthreads();
    int cur = 0, terminal = -1, bonus = 0, depth = 0;
    for (int level = 0; level <= T; ++level) {   // at most T + 1 levels
        const int n = s_count[cur];
        if (n == 0)
            break;
        if (u == 0)
            s_count[cur ^ 1] = 0;
        // the level's lowest index is the terminal if no deeper level follows
        int lo = INT_MAX;
        for (int k = 0; k < n; ++k)
            lo = min(lo, s_level[cur][k]);
        for (int k = 0; k < n; ++k) {
            const int f = s_level[cur][k];
            const int a = row_argmax<kFinThreads>(
                logits + ((size_t)b * (Tmax + 1) + (f + 1)) * V, V, shv, shi);   // ends with a barrier
            if (f == lo) {
                terminal = f;
                bonus = a;
                depth = level;
            }
            // the children of f whose token is the argmax, one thread per node
            // (in any order: the level's minimum is taken above)
            for (int c = u; c < T; c += kFinThreads)
                if (s_par[c] == f && s_tok[c] == a) {
                    const int m = atomicAdd(&s_count[cur ^ 1], 1);
                    if (in_bounds(m, kMaxTree + 1, dev_status))
                        s_level[cur ^ 1][m] = c;
                }
        }
        __syncthreads();   // the next level is complete
        cur ^= 1;
    }
    // the terminal's root path, by parent pointers, deepest first
    if (u == 0) {
        int v = terminal;
        for (int pos = depth - 1; pos >= 0 && v >= 0; --pos) {
            if (in_bounds(pos, Tmax, dev_status)) {
                out_path[(size_t)b * Tmax + pos] = v;
                out_tokens[(size_t)b * (Tmax + 1) + pos] = s_tok[v];
            }
            v = s_par[v];
        }
        if (in_bounds(depth, Tmax + 1, dev_status)) {
            out_tokens[(size_t)b * (Tmax + 1) + depth] = bonus;
            n_accepted[b] = depth;
        }
    }
}

// -------------------------------------------------------------- stochastic

// VEC: V % 4 == 0, so every logits / q row is 16-byte aligned (the entry
// point checks the base pointers) and the passes use float4 loads.
// Grid: teams x K CTAs; team t walks sequences t, t + teams, ...
// CLUSTER: a team is a thread-block cluster of K CTAs, which exchange their
// partial sums through distributed shared memory (cluster_exchange: a store
// and an mbarrier arrival per peer, then one local wait); otherwise a team is
// K CTAs of a cooperative launch exchanging them through global memory
// (per-CTA slots and an arrival counter, team_barrier).
template <bool VEC, bool CACHED, bool CLUSTER>
__global__ void __launch_bounds__(kWalkThreads, CACHED ? 3 : 4)
    mss_walk_kernel(const float *__restrict__ logits, double temp,
                    const float *__restrict__ q_probs, int Rq, const int32_t *__restrict__ q_row,
                    const int32_t *__restrict__ tokens, const int32_t *__restrict__ n_nodes,
                    const int32_t *__restrict__ first_child,
                    const int32_t *__restrict__ next_sibling,
                    const double *__restrict__ u_accept, const double *__restrict__ u_sample,
                    int B, int Tmax, int V, int K, int chunk, VerifyWs ws,
                    int32_t *__restrict__ out_tokens, int32_t *__restrict__ out_path,
                    int32_t *__restrict__ n_accepted, int32_t *dev_status)
{
    __shared__ double table[kExpTable];
    __shared__ float shf[kWalkWarps];
    __shared__ double shd[kWalkWarps];
    __shared__ int shi[kWalkWarps];
    __shared__ RowState st;
    __shared__ int sh_ok, sh_dec, sh_pick, sh_token;
    __shared__ double sh_carry;
    // the final distribution p^(n) of the current row summed over each of
    // the team's K chunks (and each chunk's largest x with p > 0): kept up to
    // date by every pass, so the draw needs no pass of its own
    __shared__ double draw_sum[32];
    __shared__ int draw_last[32];
    // the sequence's tree (child lists, tokens, q rows), staged once
    __shared__ int s_fc[kMaxTree + 1], s_ns[kMaxTree], s_tok[kMaxTree], s_qr[kMaxTree];
    // the first kDecCache children of every row (-1 past the last), so that
    // looking one up walks no sibling chain
    __shared__ int s_kid[kMaxTree + 1][kDecCache];
    // the operands of the acceptance tests of the current row's first
    // kDecCache children, loaded while the row's m/Z pass runs:
    // dc[i] = l(x_i), dc[kDecCache + i] = u_i, dc[2 kDecCache + i(i+1)/2 + j] =
    // q_j(x_i) for j <= i (q_j: the q row of child j; j = i: the child's own)
    __shared__ double dc[kDecOps];
    __shared__ unsigned long long dc_raw[kDecOps];   // their raw bits, as fetched
    // CACHED: this CTA's chunk of the current distribution, p(x) = pc[x - x_lo] * g
    __shared__ double pc[CACHED ? kCacheChunk : 1];
    __shared__ XchgShared xs;   // CLUSTER: the team's partials, in every CTA
    // STAGE (cached, 16-byte aligned rows): each pass reads its chunk from
    // shared memory, where a bulk copy put it -- for every pass after the
    // first of a sequence, issued at the start of the pass before, which
    // fetches both chunks the next pass may need (the next child's own logits
    // row and its q row), so their latency hides behind a whole pass,
    // exchange and decision.  Set n & 1 serves pass n.
    constexpr bool STAGE = CACHED && VEC;
    extern __shared__ __align__(16) float walk_stage[];   // [2 sets][logits, q][kCacheChunk]
    __shared__ __align__(8) unsigned long long stage_bar[2];
    __shared__ int stage_abort;
    double g = 0.0;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int teams = gridDim.x / K;
    const int team = blockIdx.x / K;
    const int k = CLUSTER ? (int)cluster_ctarank() : blockIdx.x % K;
    const int x_lo = min(k * chunk, V), x_hi = min(x_lo + chunk, V);
    const double inv_temp = 1.0 / temp;
    const bool lead = k == 0 && tid == 0;   // writes the path and the error codes
    int2 *tm = ws.team + team;
    int nbar = 0;
    // this CTA's slot / the team's K slots of the next barrier
    auto slots = [&]() { return ws.slot + (nbar & 1) * kWalkMaxCtas + team * K; };
    fill_exp_table(table, 1.0);   // read only from here on (barriers below publish it)
    if (STAGE) {
        if (tid == 0) {
            ptx::mbar_init(ptx::smem_addr(&stage_bar[0]), 1);
            ptx::mbar_init(ptx::smem_addr(&stage_bar[1]), 1);
            stage_abort = 0;
            ptx::fence_barrier_init();
        }
        __syncthreads();
    }
    // per set: a copy in flight (pending), the sources it holds, and the
    // phases of its barrier waited for (the same in every thread)
    bool pending0 = false, pending1 = false;
    const float *have_l0 = nullptr, *have_l1 = nullptr, *have_q0 = nullptr, *have_q1 = nullptr;
    int waits0 = 0, waits1 = 0, npass = 0;
    const uint32_t stage_bytes = (uint32_t)(x_hi - x_lo) * 4u;
    // thread 0: copy this CTA's chunks of the rows lsrc / qsrc (either may be
    // null) into set `set`; every thread has finished reading that set
    auto stage_issue = [&](int set, const float *lsrc, const float *qsrc) {
        const uint32_t bar = ptx::smem_addr(&stage_bar[set]);
        const uint32_t dst = ptx::smem_addr(walk_stage + set * 2 * kCacheChunk);
        ptx::fence_proxy_async_smem();   // the set's earlier reads before the copy's writes
        ptx::mbar_arrive_expect_tx(bar, stage_bytes * ((lsrc ? 1u : 0u) + (qsrc ? 1u : 0u)));
        if (lsrc && stage_bytes)
            ptx::bulk_load(dst, lsrc + x_lo, stage_bytes, bar);
        if (qsrc && stage_bytes)
            ptx::bulk_load(dst + 4u * kCacheChunk, qsrc + x_lo, stage_bytes, bar);
    };
    // every thread: wait for set `set` (bounded); false on timeout
    auto stage_wait = [&](int set) {
        int &w = set ? waits1 : waits0;
        const bool ok = ptx::mbar_wait(ptx::smem_addr(&stage_bar[set]), (uint32_t)(w & 1),
                                       &stage_abort, kTeamWaitNs);
        ++w;
        (set ? pending1 : pending0) = false;
        return ok;
    };
    // Start of a pass that reads row `need` (a logits row, or a q row if
    // is_q), followed by a decision on the child whose own logits row and q
    // row are next_l and next_q (null: no decision on a child follows):
    // returns the chunk to read (the global row when not staging), nullptr
    // on timeout.
    auto stage_pass = [&](const float *need, bool is_q, const float *next_l, const float *next_q)
        -> const float * {
        if (!STAGE)
            return need;
        const int set = npass & 1;
        ++npass;
        bool &pend = set ? pending1 : pending0;
        const float *&hl = set ? have_l1 : have_l0;
        const float *&hq = set ? have_q1 : have_q0;
        bool ok = true;
        if (pend && (is_q ? hq : hl) != need) {   // staged for another outcome: drain
            ok = stage_wait(set);
        }
        __syncthreads();   // every thread is done with the other set (the pass before)
        if (tid == 0) {
            if (!pend)
                stage_issue(set, is_q ? nullptr : need, is_q ? need : nullptr);
            if (next_l)
                stage_issue(set ^ 1, next_l, next_q);
        }
        if (!pend) {
            hl = is_q ? nullptr : need;
            hq = is_q ? need : nullptr;
            pend = true;
        }
        if (next_l) {
            (set ? pending0 : pending1) = true;
            (set ? have_l0 : have_l1) = next_l;
            (set ? have_q0 : have_q1) = next_q;
        }
        ok = stage_wait(set) && ok;
        if (!__syncthreads_and(ok))
            return nullptr;
        return walk_stage + set * 2 * kCacheChunk + (is_q ? kCacheChunk : 0);
    };
    // the team's first root row is staged while the rest is set up (a
    // sequence that turns out malformed leaves it pending: the next pass
    // drains it)
    if (STAGE && team < B) {
        const float *root = logits + (size_t)team * (Tmax + 1) * V;
        if (tid == 0)
            stage_issue(0, root, nullptr);
        pending0 = true;
        have_l0 = root;
    }
    if (CLUSTER) {
        xchg_init(&xs, K);
        cluster_sync_all();
    }
    // Publish this CTA's partial v and wait for the team's K partials: their
    // array (nullptr when the wait ran out, on every thread of the CTA).
    auto exchange = [&](double2 v) -> const double2 * {
        if (CLUSTER) {
            const int n = nbar++;
            return cluster_exchange(&xs, K, n, v, kTeamWaitNs) ? xs.slot[n & 1] : nullptr;
        }
        double2 *sl = slots();
        if (tid == 0)
            sl[k] = v;
        ++nbar;
        return team_barrier(tm, nbar * K, &sh_ok, kTeamWaitNs) ? sl : nullptr;
    };
    // partial `i` of the last exchange (global slots bypass L1: other CTAs
    // wrote them)
    auto partial = [&](const double2 *sl, int i) { return CLUSTER ? sl[i] : __ldcg(sl + i); };

    for (int b = team; b < B; b += teams) {
        int T;
        if (!sequence_ok(n_nodes, first_child, b, Tmax, T)) {
            if (lead)
                n_accepted[b] = -1;
            continue;
        }
        int bad = 0;
        for (int u = tid; u <= T; u += kWalkThreads) {
            s_fc[u] = first_child[(size_t)b * (Tmax + 1) + u];
            if (u == T)
                break;
            const int x = tokens[(size_t)b * Tmax + u];
            const int qr = q_row[(size_t)b * Tmax + u];
            s_tok[u] = x;
            s_qr[u] = qr;
            s_ns[u] = next_sibling[(size_t)b * Tmax + u];
            bad |= (x < 0 || x >= V) ? TSD_DEV_BAD_TOKEN : 0;
            bad |= (qr < 0 || qr >= Rq) ? TSD_DEV_BAD_QROW : 0;
        }
        if (__syncthreads_or(bad)) {   // the same answer in every CTA of the team
            if (k == 0 && bad)
                flag(dev_status, bad);
            if (lead)
                n_accepted[b] = -1;
            continue;
        }
        for (int u = tid; u <= T; u += kWalkThreads) {
            int c = s_fc[u];
#pragma unroll
            for (int i = 0; i < kDecCache; ++i) {
                s_kid[u][i] = c;
                c = (c >= 0 && c < T) ? s_ns[c] : -1;
            }
        }
        __syncthreads();
        // child i (ascending index) of the node whose logits row is `row`; -1
        // past the last (the lists come from the mask build: they are
        // increasing and inside the tree)
        auto child = [&](int row, int i) {
            int c = s_kid[row][min(i, kDecCache - 1)];
            for (i -= kDecCache - 1; c >= 0 && i > 0; --i)
                c = (c < T) ? s_ns[c] : -1;
            return (c >= 0 && in_bounds(c, T, dev_status)) ? c : -1;
        };
        auto qrow = [&](int c) { return q_probs + ((size_t)b * Rq + s_qr[c]) * V; };
        int row = 0, n_path = 0;
        bool alive = true;
        for (;;) {
            const size_t ri = (size_t)b * (Tmax + 1) + row;
            const float *lrow = logits + ri * V;
            int op = -1;
            // exp((l(x_c) - m) / T) of child i, on every lane of warp 0 (it
            // needs the row's max only, so it runs beside the sum's reduction)
            auto test_exp = [&](int i, int c, double m) {
                const double lx = i < kDecCache ? dc[i] : (double)lrow[s_tok[c]];
                return exp((lx - m) * inv_temp);
            };
            // lane 0 of warp 0: the acceptance test of child i from its
            // test_exp value e, given the row's 1/Z and the i siblings
            // rejected before it (in st)
            auto accept = [&](int i, int c, double e, double inv_Z) {
                const int x = s_tok[c];
                double qx, u;
                if (i < kDecCache) {
                    u = dc[kDecCache + i];
                    qx = dc[2 * kDecCache + i * (i + 1) / 2 + i];
                } else {
                    u = u_accept[(size_t)b * Tmax + c];
                    qx = (double)qrow(c)[x];
                }
                double p = e * inv_Z;
                for (int j = 0; j < st.n; ++j) {
                    if (st.S[j] > 0.0) {
                        const double qj = i < kDecCache
                                              ? dc[2 * kDecCache + i * (i + 1) / 2 + j]
                                              : (double)st.q[j][x];
                        const double r = p - qj;
                        p = (r > 0.0 ? r : 0.0) * st.inv_S[j];
                    }
                }
                return (p > 0.0 && u * qx <= p) ? 1 : 0;
            };
            // Without staging: the next pass reads this CTA's chunk of the
            // first child's own logits row (if it is accepted) or of its q
            // row (if not); start fetching both into L2 now, behind this pass
            // and the exchange.
            auto prefetch_next = [&](int c) {
                if (VEC && tid == 0 && c >= 0 && x_hi > x_lo) {
                    const uint32_t bytes = (uint32_t)(x_hi - x_lo) * 4u;
                    prefetch_l2(logits + ((size_t)b * (Tmax + 1) + c + 1) * V + x_lo, bytes);
                    prefetch_l2(qrow(c) + x_lo, bytes);
                }
            };
            auto lrow_of = [&](int c) {
                return logits + ((size_t)b * (Tmax + 1) + c + 1) * V;
            };
            const int c0 = child(row, 0);
            if (!STAGE)
                prefetch_next(c0);
            const float *lsrc = stage_pass(lrow, false, c0 >= 0 ? lrow_of(c0) : nullptr,
                                           c0 >= 0 ? qrow(c0) : nullptr);
            if (!lsrc) {
                alive = false;
                break;
            }
            // fetch the acceptance-test operands (read after the pass below)
            // by asynchronous copies into shared memory, which no barrier of
            // the pass waits for; operand t on thread 4t (at most eight
            // scattered loads per warp)
            if ((tid & 3) == 0 && (tid >> 2) < kDecOps) {
                const int t = tid >> 2;
                int i = -1, j = -1;
                if (t < kDecCache)
                    i = t;
                else if (t < 2 * kDecCache)
                    i = t - kDecCache;
                else {
                    const int t2 = t - 2 * kDecCache;   // i (i + 1) / 2 + j, j <= i
                    i = (int)((sqrtf(8.f * (float)t2 + 1.f) - 1.f) * 0.5f);
                    i += ((i + 1) * (i + 2) / 2 <= t2) - (i * (i + 1) / 2 > t2);
                    j = t2 - i * (i + 1) / 2;
                }
                const int ci = child(row, i);
                if (ci >= 0) {
                    const int x = s_tok[ci];
                    const uint32_t dst = ptx::smem_addr(&dc_raw[t]);
                    if (t < kDecCache) {
                        cp_async4(dst, lrow + x);
                    } else if (t < 2 * kDecCache) {
                        cp_async8(dst, u_accept + (size_t)b * Tmax + ci);
                    } else {
                        const int cj = child(row, j);
                        cp_async4(dst, qrow(cj) + x);
                    }
                    op = t;
                }
            }
            // m and Z of this row (slot: z_k, then m_k as fp32 bits | last_k)
            int lastk;
            const double2 mz =
                CACHED ? chunk_max_z_cached<VEC, STAGE>(lsrc, x_lo, x_hi, V, inv_temp, table, pc,
                                                        shf, shd, shi, &lastk)
                       : chunk_max_z<VEC>(lrow, x_lo, x_hi, V, inv_temp, table, shf, shd, shi,
                                          &lastk);
            if (op >= 0) {   // long arrived: the pass took longer than the fetch
                cp_async_wait_all();
                const unsigned long long raw = dc_raw[op];
                dc[op] = (op >= kDecCache && op < 2 * kDecCache)
                             ? __longlong_as_double((long long)raw)
                             : (double)__uint_as_float((uint32_t)raw);
            }
            const double2 *sl =
                exchange(make_double2(mz.y, __hiloint2double(__float_as_int((float)mz.x), lastk)));
            if (!sl) {
                alive = false;
                break;
            }
            int c = child(row, 0);   // the children in ascending index
            if (warp == 0) {
                double mk = -INFINITY, zk = 0.0;
                int lk = -1;
                if (lane < K) {
                    const double2 v = partial(sl, lane);
                    zk = v.x;
                    mk = (double)__int_as_float(__double2hiint(v.y));
                    lk = __double2loint(v.y);
                }
                double m = mk;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
                const double e0 = c >= 0 ? test_exp(0, c, m) : 0.0;
                const double zs =
                    mk == -INFINITY ? 0.0 : zk * table_exp((mk - m) * inv_temp, table);
                const double Z = warp_sum(zs);
                const double inv_Z = 1.0 / Z;
                draw_sum[lane] = zs * inv_Z;
                draw_last[lane] = lk;
                if (lane == 0) {
                    st.m = m;
                    st.Z = Z;
                    st.inv_Z = inv_Z;
                    st.temp = temp;
                    st.inv_temp = inv_temp;
                    st.n = 0;
                    sh_dec = c >= 0 ? accept(0, c, e0, inv_Z) : 0;
                }
            }
            __syncthreads();
            if (CACHED)   // every thread: this CTA's scale of its cached chunk
                g = mz.x == -INFINITY
                        ? 0.0
                        : table_exp((mz.x - st.m) * inv_temp, table) * st.inv_Z;
            int accepted = -1;
            for (int i = 0; c >= 0; ++i) {
                if (sh_dec) {
                    accepted = c;
                    break;
                }
                const float *qc = qrow(c);
                const int nx = child(row, i + 1);   // the sibling tested next
                if (!STAGE)
                    prefetch_next(nx);
                const float *qsrc = stage_pass(qc, true, nx >= 0 ? lrow_of(nx) : nullptr,
                                               nx >= 0 ? qrow(nx) : nullptr);
                if (!qsrc) {
                    alive = false;
                    break;
                }
                const double s =
                    CACHED ? chunk_residual_cached<VEC, STAGE>(qsrc, x_lo, x_hi, V, pc, g, shd, shi,
                                                               &lastk)
                           : chunk_residual<VEC>(lrow, qc, x_lo, x_hi, V, st, table, shd, shi,
                                                 &lastk);
                sl = exchange(make_double2(s, (double)lastk));
                if (!sl) {
                    alive = false;
                    break;
                }
                const int next = child(row, i + 1);
                if (warp == 0) {
                    double sk = 0.0;
                    int lk = -1;
                    if (lane < K) {
                        const double2 v = partial(sl, lane);
                        sk = v.x;
                        lk = (int)v.y;
                    }
                    const double en = next >= 0 ? test_exp(i + 1, next, st.m) : 0.0;
                    const double S = warp_sum(sk);
                    const double inv_S = S > 0.0 ? 1.0 / S : 0.0;
                    if (S > 0.0) {   // else p stays as it was
                        draw_sum[lane] = sk * inv_S;
                        draw_last[lane] = lk;
                    }
                    if (lane == 0) {
                        st.q[st.n] = qc;
                        st.S[st.n] = S;
                        st.inv_S[st.n] = inv_S;
                        st.n += 1;
                        sh_dec = next >= 0 ? accept(i + 1, next, en, st.inv_Z) : 0;
                    }
                }
                __syncthreads();
                if (CACHED && st.S[st.n - 1] > 0.0) {   // else p stays as it was
                    chunk_renormalise_cached<VEC, STAGE>(qsrc, x_lo, x_hi, V, pc, g,
                                                         st.inv_S[st.n - 1]);
                    g = 1.0;
                }
                c = next;
            }
            if (!alive)
                break;
            if (accepted >= 0 && n_path < T) {
                if (lead && in_bounds(n_path, Tmax, dev_status)) {
                    out_path[(size_t)b * Tmax + n_path] = accepted;
                    out_tokens[(size_t)b * (Tmax + 1) + n_path] = s_tok[accepted];
                }
                ++n_path;
                row = accepted + 1;
                continue;
            }
            // The walk stops here: draw the final token from p^(n), first
            // the chunk (from the sums the last pass left), then the token.
            const double u = u_sample[ri];
            if (warp == 0) {
                const double sk = draw_sum[lane];
                const int lk = draw_last[lane];
                double incl = sk;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const double y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o)
                        incl += y;
                }
                double excl = __shfl_up_sync(0xffffffffu, incl, 1);
                if (lane == 0)
                    excl = 0.0;
                const unsigned hit = __ballot_sync(0xffffffffu, lane < K && excl + sk > u);
                int lmax = lk;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
                const int pick = hit ? __ffs(hit) - 1 : -1;
                const double carry = __shfl_sync(0xffffffffu, excl, pick >= 0 ? pick : 0);
                const int lpick = __shfl_sync(0xffffffffu, lk, pick >= 0 ? pick : 0);
                if (lane == 0) {
                    sh_pick = pick;
                    sh_carry = carry;
                    sh_token = pick >= 0 ? lpick : lmax;
                }
            }
            __syncthreads();
            const int pick = sh_pick;
            if (pick == k) {
                int token = CACHED ? chunk_scan_cached(pc, g, x_lo, x_hi, sh_carry, u, shd, shi)
                                   : chunk_scan<VEC>(lrow, x_lo, x_hi, V, st, table, sh_carry, u,
                                                     shd, shi);
                if (token == INT_MAX)   // the chunk's own sum fell short by rounding
                    token = sh_token;
                if (tid == 0 && in_bounds(n_path, Tmax + 1, dev_status)) {
                    out_tokens[(size_t)b * (Tmax + 1) + n_path] = token;
                    n_accepted[b] = n_path;
                }
            } else if (pick < 0 && k == 0 && tid == 0 && in_bounds(n_path, Tmax + 1, dev_status)) {
                // Rounding left the total at or below u: the largest token with p > 0.
                out_tokens[(size_t)b * (Tmax + 1) + n_path] = sh_token;
                n_accepted[b] = n_path;
            }
            break;
        }
        if (!alive) {
            if (tid == 0)
                flag(dev_status, TSD_DEV_TIMEOUT);
            if (lead)
                for (int bb = b; bb < B; bb += teams)
                    n_accepted[bb] = -1;
            break;
        }
    }
    if (STAGE) {   // copies still in flight (a walk that gave up): let them land
        if (pending0)
            stage_wait(0);
        if (pending1)
            stage_wait(1);
    }
    if (CLUSTER)   // no CTA leaves while a peer may still store to it
        cluster_sync_all();
}

}  // namespace

size_t verify_workspace(int B, int Tmax, int V)
{
    (void)V;
    return kWalkBytes + align256((size_t)B * (Tmax + 1) * sizeof(int32_t));
}

size_t verify_stochastic_scratch() { return kWalkBytes; }

// The greedy form.  The all-rows scan (every row with children, then a
// finalize pass) reads up to B (Tmax + 1) V floats at HBM speed, in time
// that grows with the batch; the matched-path walk reads the root row and
// the matched nodes' rows, one CTA per sequence, in time that does not (a
// few microseconds a level).  So the walk takes batches whose scan would
// read at least kGreedyWalkBytes, the scan the smaller ones.  Side by side
// with the stochastic walk the scan's traffic also lengthens the latter's
// dependent fetches, which the walk avoids.  TSD_GREEDY_FORM = "walk" or
// "rows" forces a form (read at every launch).
constexpr double kGreedyWalkBytes = 64.0 * 1024 * 1024;

bool greedy_all_rows(int B, int Tmax, int V)
{
    if (const char *e = std::getenv("TSD_GREEDY_FORM")) {
        if (std::strcmp(e, "rows") == 0)
            return true;
        if (std::strcmp(e, "walk") == 0)
            return false;
    }
    return (double)B * (Tmax + 1) * V * sizeof(float) < kGreedyWalkBytes;
}

int launch_verify_greedy(const float *logits, const int32_t *tokens, const int32_t *parent,
                         const int32_t *n_nodes, const uint32_t *mask,
                         const int32_t *first_child, int B, int Tmax, int V,
                         int32_t *out_tokens, int32_t *out_path, int32_t *n_accepted, void *ws,
                         int32_t *dev_status, cudaStream_t stream)
{
    if (B == 0)
        return TSD_OK;
    if (!greedy_all_rows(B, Tmax, V)) {
        greedy_walk_kernel<<<B, kFinThreads, 0, stream>>>(logits, tokens, parent, n_nodes,
                                                          first_child, Tmax, V, out_tokens,
                                                          out_path, n_accepted, dev_status);
        TSD_LAUNCH_CHECK();
        return TSD_OK;
    }
    const VerifyWs w = carve(ws);
    greedy_rows_kernel<<<dim3(Tmax + 1, B), kRowThreads, 0, stream>>>(logits, n_nodes,
                                                                      first_child, Tmax, V,
                                                                      w.argmax);
    TSD_LAUNCH_CHECK();
    greedy_finalize_kernel<<<B, kFinThreads, 0, stream>>>(
        logits, tokens, parent, n_nodes, mask, first_child, Tmax, V, w.argmax, out_tokens,
        out_path, n_accepted, dev_status);
    TSD_LAUNCH_CHECK();
    return TSD_OK;
}

namespace {

// The cluster form always keeps its chunks in shared memory.
const void *walk_kernel(bool vec, bool cached, bool cluster)
{
    if (cluster)
        return vec ? reinterpret_cast<const void *>(mss_walk_kernel<true, true, true>)
                   : reinterpret_cast<const void *>(mss_walk_kernel<false, true, true>);
    return vec ? (cached ? reinterpret_cast<const void *>(mss_walk_kernel<true, true, false>)
                         : reinterpret_cast<const void *>(mss_walk_kernel<true, false, false>))
               : (cached ? reinterpret_cast<const void *>(mss_walk_kernel<false, true, false>)
                         : reinterpret_cast<const void *>(mss_walk_kernel<false, false, false>));
}

// Dynamic shared memory of a walk instance: the staged chunks of the cached
// form over 16-byte aligned rows.
int walk_smem(bool vec, bool cached) { return (vec && cached) ? kStageBytes : 0; }

// The dynamic shared-memory limit of every walk instance that stages, set
// once per device (a function attribute of the current device).
bool walk_attributes()
{
    constexpr int kMaxDevices = 64;
    static std::atomic<int> done[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return false;
    if (done[dev].load(std::memory_order_acquire))
        return true;
    const void *fns[] = {walk_kernel(true, true, false), walk_kernel(true, true, true)};
    bool ok = true;
    for (const void *fn : fns)
        ok = ok && cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kStageBytes) == cudaSuccess;
    if (!ok) {
        (void)cudaGetLastError();
        return false;
    }
    done[dev].store(1, std::memory_order_release);
    return true;
}

// CTAs of the walk kernel that fit on the device at once (the cooperative
// launch limit), capped by the workspace slots; looked up once per device.
// The cluster form is sized by the same per-SM occupancy.
int walk_capacity(bool vec, bool cached)
{
    // Threads making their first call on a device at the same time may both
    // compute the value (the same one); the atomic makes that race benign.
    constexpr int kMaxDevices = 64;
    static std::atomic<int> cap[2][2][kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return 0;
    std::atomic<int> &slot = cap[vec ? 1 : 0][cached ? 1 : 0][dev];
    int c = slot.load(std::memory_order_relaxed);
    if (c == 0) {
        int sms = 0, occ = 0, coop = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
        const void *fn = walk_kernel(vec, cached, false);
        if (!walk_attributes())
            return 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kWalkThreads,
                                                      walk_smem(vec, cached));
        (void)cudaGetLastError();
        c = coop ? std::min(sms * occ, kWalkMaxCtas) : -1;
        slot.store(c, std::memory_order_relaxed);
    }
    return c;
}

// Grid of the walk for B sequences over a vocabulary of V on the current
// device.  Team size: enough CTAs that each owns at least kTeamMinChunk
// entries (at most kTeamMax), as long as every sequence still gets a team;
// with more sequences than the grid holds, one-CTA teams each walk several.
int walk_grid_for(int cap, int B, int V, int &K, int &teams, int &chunk)
{
    if (cap <= 0 || B < 1)
        return TSD_ERR_CUDA;
    const int k_want = std::max(1, std::min(kTeamMax, V / kTeamMinChunk));
    if ((long)B * k_want <= cap) {
        K = k_want;
        teams = B;
    } else {
        K = std::max(1, cap / B);
        teams = std::min(B, cap / K);
    }
    chunk = (V + K - 1) / K;
    chunk = (chunk + 3) & ~3;
    return TSD_OK;
}

// TSD_WALK_EXCHANGE=global keeps the cooperative form where the cluster form
// applies (read at every launch; for A/B runs and the tests).
bool walk_global_forced()
{
    const char *e = getenv("TSD_WALK_EXCHANGE");
    return e && strcmp(e, "global") == 0;
}

// The walk plan.  Cluster form: a vocabulary of at most kClusterTeam x
// kCacheChunk entries, split over K <= kClusterTeam CTAs of one cluster
// (K = V / kTeamMinChunk rounded up, so that each CTA's chunk of the current
// distribution stays in its shared memory); a team per sequence as long as
// the teams fit on the device at once, else fewer teams that each walk
// several sequences (clusters need no co-residency with each other).
// Otherwise the cooperative form; it keeps each CTA's chunk in shared memory
// (`cached`) when the chunk fits kCacheChunk entries, else it recomputes the
// distribution from the rows in every pass.
int walk_grid(int B, int V, int &K, int &teams, int &chunk, bool &cached, bool &cluster)
{
    const bool vec = (V & 3) == 0;
    cluster = !walk_global_forced() && (long)V <= (long)kClusterTeam * kCacheChunk;
    if (cluster) {
        const int cap = walk_capacity(vec, true);
        if (cap <= 0 || B < 1)
            return TSD_ERR_CUDA;
        K = std::max(1, std::min(kClusterTeam, (V + kTeamMinChunk - 1) / kTeamMinChunk));
        chunk = (((V + K - 1) / K) + 3) & ~3;
        if (chunk > kCacheChunk) {   // V just below the limit: the largest team
            K = kClusterTeam;
            chunk = (((V + K - 1) / K) + 3) & ~3;
        }
        teams = std::max(1, std::min(B, cap / K));
        cached = true;
        return TSD_OK;
    }
    int rc = walk_grid_for(walk_capacity(vec, true), B, V, K, teams, chunk);
    cached = rc == TSD_OK && chunk <= kCacheChunk;
    if (!cached)
        rc = walk_grid_for(walk_capacity(vec, false), B, V, K, teams, chunk);
    return rc;
}

}  // namespace

int verify_stochastic_plan(int B, int V, int32_t out[4])
{
    int K, teams, chunk;
    bool cached, cluster;
    const int rc = walk_grid(B, V, K, teams, chunk, cached, cluster);
    if (rc != TSD_OK)
        return rc;
    out[0] = teams;
    out[1] = K;
    out[2] = chunk;
    out[3] = teams * K;
    return TSD_OK;
}

int launch_verify_stochastic(const float *logits, double temperature, const float *q_probs,
                             int Rq, const int32_t *q_row, const int32_t *tokens,
                             const int32_t *n_nodes, const int32_t *first_child,
                             const int32_t *next_sibling, const double *u_accept,
                             const double *u_sample, int B, int Tmax, int V,
                             int32_t *out_tokens, int32_t *out_path, int32_t *n_accepted,
                             void *ws, int32_t *dev_status, cudaStream_t stream)
{
    if (B == 0)
        return TSD_OK;
    const bool vec = (V & 3) == 0;
    int K, teams, chunk;
    bool cached, cluster;
    if (walk_grid(B, V, K, teams, chunk, cached, cluster) != TSD_OK)
        return TSD_ERR_CUDA;
    VerifyWs w = carve(ws);
    if (!cluster && cudaMemsetAsync(w.team, 0, (size_t)teams * sizeof(int2), stream) != cudaSuccess) {
        (void)cudaGetLastError();
        return TSD_ERR_CUDA;
    }
    void *args[] = {(void *)&logits,      (void *)&temperature, (void *)&q_probs,
                    (void *)&Rq,          (void *)&q_row,       (void *)&tokens,
                    (void *)&n_nodes,     (void *)&first_child, (void *)&next_sibling,
                    (void *)&u_accept,    (void *)&u_sample,    (void *)&B,
                    (void *)&Tmax,        (void *)&V,           (void *)&K,
                    (void *)&chunk,       (void *)&w,           (void *)&out_tokens,
                    (void *)&out_path,    (void *)&n_accepted,  (void *)&dev_status};
    const void *fn = walk_kernel(vec, cached, cluster);
    const int smem = walk_smem(vec, cached);
    if (smem && !walk_attributes())
        return TSD_ERR_CUDA;
    cudaError_t err;
    if (cluster) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(teams * K);
        cfg.blockDim = dim3(kWalkThreads);
        cfg.dynamicSmemBytes = (size_t)smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)K;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        err = cudaLaunchKernelExC(&cfg, fn, args);
    } else {
        err = cudaLaunchCooperativeKernel(fn, dim3(teams * K), dim3(kWalkThreads), args,
                                          (size_t)smem, stream);
    }
    if (err != cudaSuccess) {
        (void)cudaGetLastError();
        return TSD_ERR_CUDA;
    }
    TSD_LAUNCH_CHECK();
    return TSD_OK;
}

}  // namespace tsd
