// Tree verification from the target model's logits (SpecInfer explainer,
// section "ツリー検証アルゴリズム").
//
// greedy
//   greedy_rows_kernel      one CTA per logits row whose node has children:
//                           argmax (lowest index on ties), float4 loads, several
//                           in flight per thread;
//   greedy_finalize_kernel  one CTA per sequence: the nodes whose whole root
//                           path matches, the deepest (lowest index on ties),
//                           and the argmax of its row (computed here for a leaf).
// stochastic (multi-step speculative sampling)
//   mss_rows_kernel         one CTA per logits row (every node and the root):
//                           m = max l and Z = sum exp((l-m)/T) in fp64; for a
//                           row with children, the children in ascending index:
//                           child c with token x is accepted iff p(x) > 0 and
//                           u_c * q_c(x) <= p(x) (one thread, exact fp64
//                           formula); after a rejection the block computes
//                           S = sum max(0, p - q_c), and p becomes
//                           max(0, p - q_c) / S.
//   mss_chunks_kernel       one CTA per (vocabulary chunk, sequence): follows
//                           the accepted children from the root to the row where
//                           the sequence stops and sums that row's final
//                           distribution over its chunk;
//   mss_finalize_kernel     one CTA per sequence: emits the path, then draws the
//                           last token by inverse CDF at u_sample[row] -- the
//                           chunk whose running sum passes u, then an fp64
//                           block scan inside that chunk.
//
// Residual distributions are never materialised: p^(n)(x) is recomputed per
// element from the logits row, the rejected siblings' q rows and their
// normalisers.  The bulk sums (Z, S, the CDF) use a table-driven fp64 exp
// (its table pre-scaled by 1/Z) and reciprocals; the acceptance tests use the
// exact formula.  Both agree with a sequential fp64 evaluation to ~1e-15
// relative, so a decision can only differ when its uniform lies within that
// distance of the boundary.
#include <climits>

#include "fp64_exp.cuh"
#include "tsd_common.cuh"

namespace tsd {

namespace {

constexpr int kRowThreads = 512;
constexpr int kWarps = kRowThreads / 32;
constexpr int kFinThreads = 1024;
constexpr int kDrawThreads = 256;
constexpr int kChunk = 4096;   // vocabulary chunk of the deferred draw (multiple of 4)

struct VerifyWs {
    double *Z;            // [B][Tmax+1]  sum exp((l - m)/T)
    double *S;            // [B][Tmax]    residual normaliser after rejecting child c
    double *chunk_sum;    // [B][nch]     final distribution summed over a chunk
    int32_t *argmax;      // [B][Tmax+1]  greedy: argmax of rows with children
    int32_t *accepted;    // [B][Tmax+1]  accepted child per row, -1 none
    float *rmax;          // [B][Tmax+1]  row max
    int32_t *chunk_last;  // [B][nch]     largest token of the chunk with p > 0, or -1
    int nch;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int num_chunks(int V) { return (V + kChunk - 1) / kChunk; }

VerifyWs carve(void *ws, int B, int Tmax, int V)
{
    const size_t R = (size_t)B * (Tmax + 1), N = (size_t)B * Tmax;
    const size_t C = (size_t)B * num_chunks(V);
    char *p = static_cast<char *>(ws);
    VerifyWs w;
    w.nch = num_chunks(V);
    w.Z = reinterpret_cast<double *>(p);
    p += align256(R * sizeof(double));
    w.S = reinterpret_cast<double *>(p);
    p += align256(N * sizeof(double));
    w.chunk_sum = reinterpret_cast<double *>(p);
    p += align256(C * sizeof(double));
    w.argmax = reinterpret_cast<int32_t *>(p);
    p += align256(R * sizeof(int32_t));
    w.accepted = reinterpret_cast<int32_t *>(p);
    p += align256(R * sizeof(int32_t));
    w.rmax = reinterpret_cast<float *>(p);
    p += align256(R * sizeof(float));
    w.chunk_last = reinterpret_cast<int32_t *>(p);
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

__device__ float block_max(float v, float *sh)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_max(v);
    if (lane == 0)
        sh[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < kWarps ? sh[lane] : -INFINITY;
        v = warp_max(v);
        if (lane == 0)
            sh[0] = v;
    }
    __syncthreads();
    v = sh[0];
    __syncthreads();
    return v;
}

__device__ double block_sum(double v, double *sh)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    if (lane == 0)
        sh[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < kWarps ? sh[lane] : 0.0;
        v = warp_sum(v);
        if (lane == 0)
            sh[0] = v;
    }
    __syncthreads();
    v = sh[0];
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

// Row argmax (lowest index among the maxima); four float4 loads in flight.
template <int NT>
__device__ int row_argmax(const float *__restrict__ row, int V, float *shv, int *shi)
{
    float bv = -INFINITY;
    int bi = INT_MAX;
    if ((V & 3) == 0) {
        const float4 *r4 = reinterpret_cast<const float4 *>(row);
        const int n4 = V >> 2;
        int j = threadIdx.x;
        for (; j + 3 * NT < n4; j += 4 * NT) {
            float4 x[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                x[k] = __ldg(r4 + j + k * NT);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i0 = 4 * (j + k * NT);
                if (better(x[k].x, i0, bv, bi)) { bv = x[k].x; bi = i0; }
                if (better(x[k].y, i0 + 1, bv, bi)) { bv = x[k].y; bi = i0 + 1; }
                if (better(x[k].z, i0 + 2, bv, bi)) { bv = x[k].z; bi = i0 + 2; }
                if (better(x[k].w, i0 + 3, bv, bi)) { bv = x[k].w; bi = i0 + 3; }
            }
        }
        for (; j < n4; j += NT) {
            const float4 x = __ldg(r4 + j);
            const int i0 = 4 * j;
            if (better(x.x, i0, bv, bi)) { bv = x.x; bi = i0; }
            if (better(x.y, i0 + 1, bv, bi)) { bv = x.y; bi = i0 + 1; }
            if (better(x.z, i0 + 2, bv, bi)) { bv = x.z; bi = i0 + 2; }
            if (better(x.w, i0 + 3, bv, bi)) { bv = x.w; bi = i0 + 3; }
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

__device__ float row_max(const float *__restrict__ row, int V, float *sh)
{
    float m = -INFINITY;
    if ((V & 3) == 0) {
        const float4 *r4 = reinterpret_cast<const float4 *>(row);
        const int n4 = V >> 2;
        int j = threadIdx.x;
        for (; j + 3 * kRowThreads < n4; j += 4 * kRowThreads) {
            float4 x[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                x[k] = __ldg(r4 + j + k * kRowThreads);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                m = fmaxf(m, fmaxf(fmaxf(x[k].x, x[k].y), fmaxf(x[k].z, x[k].w)));
        }
        for (; j < n4; j += kRowThreads) {
            const float4 x = __ldg(r4 + j);
            m = fmaxf(m, fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
        }
    } else {
        for (int j = threadIdx.x; j < V; j += kRowThreads)
            m = fmaxf(m, __ldg(row + j));
    }
    return block_max(m, sh);
}

// Per-row state of multi-step speculative sampling.
struct RowState {
    double m, inv_temp, temp, Z;
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

// p^(n)(x) for x in [x0, x0+4) (0 beyond V) for the bulk sums.  `table` is
// the exp table pre-scaled by 1/Z (by 1 while Z itself is being summed); the
// loads of each rejected sibling's row are issued together.
template <bool VEC>
__device__ __forceinline__ void p_bulk4(const float *__restrict__ row, int x0, int V,
                                        const RowState &st, const double *table, double (&p)[4])
{
    float l[4];
    load4<VEC>(row, x0, V, l);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        p[k] = x0 + k < V ? table_exp(((double)l[k] - st.m) * st.inv_temp, table) : 0.0;
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

// sum_x max(0, p^(n)(x) - q(x)) (q == nullptr: sum_x p^(n)(x)), eight tokens
// per thread per iteration as two groups of four.
template <bool VEC>
__device__ double bulk_mass(const float *__restrict__ row, const float *__restrict__ q, int V,
                            const RowState &st, const double *table, double *sh)
{
    double s = 0.0;
    for (int x0 = 4 * threadIdx.x; x0 < V; x0 += 8 * kRowThreads) {
        const int x1 = x0 + 4 * kRowThreads;
        double p0[4], p1[4];
        p_bulk4<VEC>(row, x0, V, st, table, p0);
        p_bulk4<VEC>(row, x1, V, st, table, p1);
        if (q) {
            float q0[4], q1[4];
            load4<VEC>(q, x0, V, q0);
            load4<VEC>(q, x1, V, q1);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const double d0 = p0[k] - (double)q0[k], d1 = p1[k] - (double)q1[k];
                s += (d0 > 0.0 ? d0 : 0.0) + (d1 > 0.0 ? d1 : 0.0);
            }
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                s += p0[k] + p1[k];
        }
    }
    return block_sum(s, sh);
}

// p^(n)(x) for one acceptance test: the exact fp64 formula of the definition.
__device__ __forceinline__ double p_exact(float lx, int x, const RowState &st)
{
    double p = exp(((double)lx - st.m) / st.temp) / st.Z;
    for (int j = 0; j < st.n; ++j) {
        if (st.S[j] > 0.0) {
            const double r = p - (double)st.q[j][x];
            p = (r > 0.0 ? r : 0.0) / st.S[j];
        }
    }
    return p;
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
    __shared__ float shv[kWarps];
    __shared__ int shi[kWarps];
    const int r = blockIdx.x, b = blockIdx.y;
    int T;
    if (!sequence_ok(n_nodes, first_child, b, Tmax, T) || r > T)
        return;
    if (first_child[(size_t)b * (Tmax + 1) + r] < 0)
        return;   // leaf: its argmax is needed only if it ends the path
    const int a =
        row_argmax<kRowThreads>(logits + ((size_t)b * (Tmax + 1) + r) * V, V, shv, shi);
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
            out_path[(size_t)b * Tmax + pos] = u;
            out_tokens[(size_t)b * (Tmax + 1) + pos] = tok;
        }
    }
    const int row = t + 1;
    int bonus;
    if (first_child[(size_t)b * (Tmax + 1) + row] >= 0)
        bonus = argmax_ws[(size_t)b * (Tmax + 1) + row];
    else
        bonus = row_argmax<kFinThreads>(logits + ((size_t)b * (Tmax + 1) + row) * V, V, shv,
                                        shi);
    if (u == 0) {
        out_tokens[(size_t)b * (Tmax + 1) + n] = bonus;
        n_accepted[b] = n;
    }
}

// -------------------------------------------------------------- stochastic
// VEC: V % 4 == 0, so every logits / q row is 16-byte aligned (the entry
// point checks the base pointers) and the bulk passes use float4 loads.
template <bool VEC>
__global__ void __launch_bounds__(kRowThreads)
    mss_rows_kernel(const float *__restrict__ logits, double temp,
                    const float *__restrict__ q_probs, int Rq, const int32_t *__restrict__ q_row,
                    const int32_t *__restrict__ tokens, const int32_t *__restrict__ n_nodes,
                    const int32_t *__restrict__ first_child,
                    const int32_t *__restrict__ next_sibling,
                    const double *__restrict__ u_accept, int Tmax, int V, VerifyWs ws)
{
    __shared__ double table[kExpTable];
    __shared__ float shf[kWarps];
    __shared__ double shd[kWarps];
    __shared__ RowState st;
    __shared__ int decision;
    const int r = blockIdx.x, b = blockIdx.y;
    int T;
    if (!sequence_ok(n_nodes, first_child, b, Tmax, T) || r > T)
        return;
    fill_exp_table(table, 1.0);
    const float *row = logits + ((size_t)b * (Tmax + 1) + r) * V;
    const float mf = row_max(row, V, shf);   // its barriers also publish the table
    if (threadIdx.x == 0) {
        st.m = (double)mf;
        st.inv_temp = 1.0 / temp;
        st.temp = temp;
        st.n = 0;
    }
    __syncthreads();
    const double Z = bulk_mass<VEC>(row, nullptr, V, st, table, shd);
    const size_t ri = (size_t)b * (Tmax + 1) + r;
    if (threadIdx.x == 0) {
        st.Z = Z;
        ws.rmax[ri] = mf;
        ws.Z[ri] = Z;
    }
    int c = first_child[ri];
    if (c < 0) {
        if (threadIdx.x == 0)
            ws.accepted[ri] = -1;
        return;   // a leaf (or an empty tree's root): it only needs m and Z
    }
    fill_exp_table(table, 1.0 / Z);   // bulk_mass ended with a barrier: table is free
    __syncthreads();
    int accepted = -1;
    while (c >= 0) {
        const int x = tokens[(size_t)b * Tmax + c];
        const int qr = q_row[(size_t)b * Tmax + c];
        if (x < 0 || x >= V || qr < 0 || qr >= Rq)
            break;   // malformed; the finalize kernel reports it
        const float *qc = q_probs + ((size_t)b * Rq + qr) * V;
        if (threadIdx.x == 0) {
            const double px = p_exact(row[x], x, st);
            const double qx = (double)qc[x];
            const double u = u_accept[(size_t)b * Tmax + c];
            decision = (px > 0.0 && u * qx <= px) ? 1 : 0;
        }
        __syncthreads();
        if (decision) {
            accepted = c;
            break;
        }
        const double S = bulk_mass<VEC>(row, qc, V, st, table, shd);
        if (threadIdx.x == 0) {
            st.q[st.n] = qc;
            st.S[st.n] = S;
            st.inv_S[st.n] = S > 0.0 ? 1.0 / S : 0.0;
            st.n += 1;
            ws.S[(size_t)b * Tmax + c] = S;
        }
        __syncthreads();
        c = next_sibling[(size_t)b * Tmax + c];
    }
    if (threadIdx.x == 0)
        ws.accepted[ri] = accepted;
}

// Thread 0: walk the accepted children from the root (accepted row in shared
// memory), fill `st` with the final distribution's state at the row where the
// sequence stops, and return that row; n_out = accepted nodes.  Optionally
// writes the path.  st.n = -1 if a q row index is malformed.
__device__ int walk_to_terminal(int b, int T, int Tmax, int Rq, int V, double temp,
                                const float *__restrict__ q_probs,
                                const int32_t *__restrict__ q_row,
                                const int32_t *__restrict__ tokens,
                                const int32_t *__restrict__ first_child,
                                const int32_t *__restrict__ next_sibling, const VerifyWs &ws,
                                const int *acc, RowState &st, int &n_out,
                                int32_t *__restrict__ out_path, int32_t *__restrict__ out_tokens)
{
    int row = 0, n = 0;
    while (n < T && acc[row] >= 0) {
        const int c = acc[row];
        if (out_path) {
            out_path[(size_t)b * Tmax + n] = c;
            out_tokens[(size_t)b * (Tmax + 1) + n] = tokens[(size_t)b * Tmax + c];
        }
        row = c + 1;
        ++n;
    }
    const size_t ri = (size_t)b * (Tmax + 1) + row;
    st.m = (double)ws.rmax[ri];
    st.Z = ws.Z[ri];
    st.temp = temp;
    st.inv_temp = 1.0 / temp;
    st.n = 0;
    for (int c = first_child[ri]; c >= 0; c = next_sibling[(size_t)b * Tmax + c]) {
        const int qr = q_row[(size_t)b * Tmax + c];
        if (qr < 0 || qr >= Rq) {
            st.n = -1;
            break;
        }
        const double S = ws.S[(size_t)b * Tmax + c];
        st.q[st.n] = q_probs + ((size_t)b * Rq + qr) * V;
        st.S[st.n] = S;
        st.inv_S[st.n] = S > 0.0 ? 1.0 / S : 0.0;
        st.n += 1;
    }
    n_out = n;
    return row;
}

template <bool VEC>
__global__ void __launch_bounds__(kDrawThreads)
    mss_chunks_kernel(const float *__restrict__ logits, double temp,
                      const float *__restrict__ q_probs, int Rq,
                      const int32_t *__restrict__ q_row, const int32_t *__restrict__ tokens,
                      const int32_t *__restrict__ n_nodes,
                      const int32_t *__restrict__ first_child,
                      const int32_t *__restrict__ next_sibling, int Tmax, int V, VerifyWs ws)
{
    __shared__ double table[kExpTable];
    __shared__ double shd[kDrawThreads / 32];
    __shared__ int shi[kDrawThreads / 32];
    __shared__ int acc[kMaxTree + 1];
    __shared__ RowState st;
    __shared__ int term;
    const int ch = blockIdx.x, b = blockIdx.y;
    int T;
    if (!sequence_ok(n_nodes, first_child, b, Tmax, T))
        return;
    for (int i = threadIdx.x; i <= T; i += kDrawThreads)
        acc[i] = ws.accepted[(size_t)b * (Tmax + 1) + i];
    __syncthreads();
    if (threadIdx.x == 0) {
        int n;
        term = walk_to_terminal(b, T, Tmax, Rq, V, temp, q_probs, q_row, tokens, first_child,
                                next_sibling, ws, acc, st, n, nullptr, nullptr);
    }
    __syncthreads();
    if (st.n < 0)
        return;   // malformed; the finalize kernel reports it
    fill_exp_table(table, 1.0 / st.Z);
    __syncthreads();
    const float *row = logits + ((size_t)b * (Tmax + 1) + term) * V;
    const int x_begin = ch * kChunk, x_end = min(x_begin + kChunk, V);
    double s = 0.0;
    int last = -1;
    for (int x0 = x_begin + 4 * threadIdx.x; x0 < x_end; x0 += 4 * kDrawThreads) {
        double p[4];
        p_bulk4<VEC>(row, x0, V, st, table, p);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            s += p[k];
            if (p[k] > 0.0)
                last = x0 + k;
        }
    }
    // block reductions over kDrawThreads threads
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    s = warp_sum(s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
    if (lane == 0) {
        shd[warp] = s;
        shi[warp] = last;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double tot = 0.0;
        int lst = -1;
        for (int w2 = 0; w2 < kDrawThreads / 32; ++w2) {
            tot += shd[w2];
            lst = max(lst, shi[w2]);
        }
        ws.chunk_sum[(size_t)b * ws.nch + ch] = tot;
        ws.chunk_last[(size_t)b * ws.nch + ch] = lst;
    }
}

template <bool VEC>
__global__ void __launch_bounds__(kDrawThreads)
    mss_finalize_kernel(const float *__restrict__ logits, double temp,
                        const float *__restrict__ q_probs, int Rq,
                        const int32_t *__restrict__ q_row, const int32_t *__restrict__ tokens,
                        const int32_t *__restrict__ n_nodes,
                        const int32_t *__restrict__ first_child,
                        const int32_t *__restrict__ next_sibling,
                        const double *__restrict__ u_sample, int Tmax, int V, VerifyWs ws,
                        int32_t *__restrict__ out_tokens, int32_t *__restrict__ out_path,
                        int32_t *__restrict__ n_accepted, int32_t *dev_status)
{
    constexpr int NW = kDrawThreads / 32;
    __shared__ double table[kExpTable];
    __shared__ double warp_tot[NW];
    __shared__ int shi[NW];
    __shared__ int acc[kMaxTree + 1];
    __shared__ RowState st;
    __shared__ int term, n_path, chosen;
    __shared__ double carry0;
    const int b = blockIdx.x, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    int T;
    if (!sequence_ok(n_nodes, first_child, b, Tmax, T)) {
        if (tid == 0)
            n_accepted[b] = -1;
        return;
    }
    int bad = 0;
    if (tid < T) {
        const int x = tokens[(size_t)b * Tmax + tid];
        const int qr = q_row[(size_t)b * Tmax + tid];
        bad = (x < 0 || x >= V) ? TSD_DEV_BAD_TOKEN : 0;
        bad |= (qr < 0 || qr >= Rq) ? TSD_DEV_BAD_QROW : 0;
    }
    if (__syncthreads_or(bad)) {
        if (bad)
            flag(dev_status, bad);
        if (tid == 0)
            n_accepted[b] = -1;
        return;
    }
    for (int i = tid; i <= T; i += kDrawThreads)
        acc[i] = ws.accepted[(size_t)b * (Tmax + 1) + i];
    __syncthreads();
    if (tid == 0) {
        int n;
        term = walk_to_terminal(b, T, Tmax, Rq, V, temp, q_probs, q_row, tokens, first_child,
                                next_sibling, ws, acc, st, n, out_path, out_tokens);
        n_path = n;
        // The chunk whose running sum passes u.
        const double u = u_sample[(size_t)b * (Tmax + 1) + term];
        double C = 0.0;
        int pick = -1;
        for (int c = 0; c < ws.nch; ++c) {
            const double s = ws.chunk_sum[(size_t)b * ws.nch + c];
            if (C + s > u) {
                pick = c;
                break;
            }
            C += s;
        }
        chosen = pick;
        carry0 = C;
    }
    __syncthreads();
    const double u = u_sample[(size_t)b * (Tmax + 1) + term];
    int token;
    if (chosen < 0) {
        // Rounding left the total at or below u: the largest token with p > 0.
        int last = -1;
        for (int c = tid; c < ws.nch; c += kDrawThreads)
            last = max(last, ws.chunk_last[(size_t)b * ws.nch + c]);
        token = block_max_int<kDrawThreads>(last, shi);
    } else {
        fill_exp_table(table, 1.0 / st.Z);
        __syncthreads();
        const float *row = logits + ((size_t)b * (Tmax + 1) + term) * V;
        const int x_begin = chosen * kChunk, x_end = min(x_begin + kChunk, V);
        double carry = carry0;
        token = INT_MAX;
        for (int base = x_begin; base < x_end; base += 4 * kDrawThreads) {
            const int x0 = base + 4 * tid;
            double p[4] = {0.0, 0.0, 0.0, 0.0};
            if (x0 < x_end)
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
            for (int w2 = 0; w2 < NW; ++w2) {
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
                if (found == INT_MAX && x0 + k < x_end && C > u)
                    found = x0 + k;
            }
            found = block_min_int<kDrawThreads>(found, shi);
            if (found != INT_MAX) {
                token = found;
                break;
            }
            carry += tile;
        }
        if (token == INT_MAX)   // the chunk's own total fell short by rounding
            token = ws.chunk_last[(size_t)b * ws.nch + chosen];
    }
    if (tid == 0) {
        out_tokens[(size_t)b * (Tmax + 1) + n_path] = token;
        n_accepted[b] = n_path;
    }
}

}  // namespace

size_t verify_workspace(int B, int Tmax, int V)
{
    const size_t R = (size_t)B * (Tmax + 1), N = (size_t)B * Tmax;
    const size_t C = (size_t)B * num_chunks(V);
    return align256(R * sizeof(double)) + align256(N * sizeof(double)) +
           align256(C * sizeof(double)) + 3 * align256(R * sizeof(int32_t)) +
           align256(C * sizeof(int32_t));
}

int launch_verify_greedy(const float *logits, const int32_t *tokens, const int32_t *parent,
                         const int32_t *n_nodes, const uint32_t *mask,
                         const int32_t *first_child, int B, int Tmax, int V,
                         int32_t *out_tokens, int32_t *out_path, int32_t *n_accepted, void *ws,
                         int32_t *dev_status, cudaStream_t stream)
{
    if (B == 0)
        return TSD_OK;
    const VerifyWs w = carve(ws, B, Tmax, V);
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
    const VerifyWs w = carve(ws, B, Tmax, V);
    const bool vec = (V & 3) == 0;
    const dim3 rows(Tmax + 1, B), chunks(w.nch, B);
    if (vec)
        mss_rows_kernel<true><<<rows, kRowThreads, 0, stream>>>(
            logits, temperature, q_probs, Rq, q_row, tokens, n_nodes, first_child, next_sibling,
            u_accept, Tmax, V, w);
    else
        mss_rows_kernel<false><<<rows, kRowThreads, 0, stream>>>(
            logits, temperature, q_probs, Rq, q_row, tokens, n_nodes, first_child, next_sibling,
            u_accept, Tmax, V, w);
    TSD_LAUNCH_CHECK();
    if (vec)
        mss_chunks_kernel<true><<<chunks, kDrawThreads, 0, stream>>>(
            logits, temperature, q_probs, Rq, q_row, tokens, n_nodes, first_child, next_sibling,
            Tmax, V, w);
    else
        mss_chunks_kernel<false><<<chunks, kDrawThreads, 0, stream>>>(
            logits, temperature, q_probs, Rq, q_row, tokens, n_nodes, first_child, next_sibling,
            Tmax, V, w);
    TSD_LAUNCH_CHECK();
    if (vec)
        mss_finalize_kernel<true><<<B, kDrawThreads, 0, stream>>>(
            logits, temperature, q_probs, Rq, q_row, tokens, n_nodes, first_child, next_sibling,
            u_sample, Tmax, V, w, out_tokens, out_path, n_accepted, dev_status);
    else
        mss_finalize_kernel<false><<<B, kDrawThreads, 0, stream>>>(
            logits, temperature, q_probs, Rq, q_row, tokens, n_nodes, first_child, next_sibling,
            u_sample, Tmax, V, w, out_tokens, out_path, n_accepted, dev_status);
    TSD_LAUNCH_CHECK();
    return TSD_OK;
}

}  // namespace tsd
