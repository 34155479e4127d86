// Token-tree construction (SpecInfer explainer, "マルチドラフトモデルアプローチ":
// item 1, an expansion-based tree <k_1, ..., k_n> takes one SSM's top-k_i
// tokens at every node of depth i-1; item 2, a merge-based tree merges the
// outputs of several SSMs into one token tree; "Tree Attention のカーネル融合",
// item 2: the tree is laid out depth-first).
//
//   tree_expand_kernel        one CTA per (frontier node, sequence): the k best
//                             tokens of the node's SSM row (descending
//                             probability, lower token id on ties).  k <= 8:
//                             one pass (8 loads in flight per thread), each
//                             thread keeping its best k in registers, then k
//                             block arg-best rounds over the threads' lists;
//                             k > 8: k block passes, each taking the best
//                             element strictly after the previous pick in
//                             that order.  Writes the children at
//                             n_nodes + i*k + j;
//   tree_expand_commit_kernel one thread per sequence: n_nodes and lvl_begin
//                             advance once every CTA has read them;
//   tree_dfs_kernel           one thread per sequence: child lists in index
//                             order, then a stackless pre-order walk;
//   tree_merge_kernel         one thread per sequence: trie insertion of the
//                             chains (children kept in creation order), then
//                             the same pre-order walk.
// The per-sequence work is at most TSD_MAX_TREE nodes; it runs in shared
// memory, one sequence per CTA.
#include <climits>

#include "tsd_common.cuh"

namespace tsd {

namespace {

constexpr int kExpandThreads = 512;
constexpr int kLoadBatch = 8;       // loads in flight per thread in the row scans
constexpr int kMergeStage = 1024;   // chain entries staged in shared memory

// (v, i) comes before (w, j) in "descending probability, lower token first".
__device__ __forceinline__ bool before(float v, int i, float w, int j)
{
    return v > w || (v == w && i < j);
}

// Validation of one level (the commit kernel's; the expansion kernel makes the
// same checks in parallel): frontier size F, or 0 if the level cannot be
// added.
__device__ int expand_frontier(const int32_t *__restrict__ frow, int Rq, int V, int k,
                               const int32_t *__restrict__ n_nodes,
                               const int32_t *__restrict__ lvl_begin, int b, int Tmax, int &n,
                               int &lb)
{
    n = n_nodes[b];
    lb = lvl_begin[b];
    const int F = n == 0 ? 1 : n - lb;
    if (n < 0 || n > Tmax || k < 1 || k > V || F < 1 || lb < 0 || (long)n + (long)F * k > Tmax)
        return 0;
    for (int i = 0; i < F; ++i) {
        const int r = frow[(size_t)b * Tmax + i];
        if (r < 0 || r >= Rq)
            return 0;
    }
    return F;
}

// Block arg-best of (v, i) over the CTA (value desc, index asc; INT_MAX =
// none); the result in every thread.
__device__ __forceinline__ void block_best(float &v, int &i, float *shv, int *shi)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (oi != INT_MAX && (i == INT_MAX || before(ov, oi, v, i))) {
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
        v = lane < kExpandThreads / 32 ? shv[lane] : -INFINITY;
        i = lane < kExpandThreads / 32 ? shi[lane] : INT_MAX;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, v, o);
            const int oi = __shfl_xor_sync(0xffffffffu, i, o);
            if (oi != INT_MAX && (i == INT_MAX || before(ov, oi, v, i))) {
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

// The k <= KM best entries of a row (descending probability, lower token id
// on ties) in one pass: every thread keeps its own best KM in registers,
// sorted, inserting each element with a branch-free compare-and-shift (no
// divergence however often lanes insert); then k rounds of a block arg-best
// over the threads' list heads, the winner popping its head.  `emit(j, x)`
// is called by thread 0 with the j-th best token.
template <int KM, typename Emit>
__device__ __forceinline__ void row_topk_one_pass(const float *__restrict__ p, int V, bool vec,
                                                  int k, float *shv, int *shi, Emit emit)
{
    float lv[KM];
    int li[KM];
#pragma unroll
    for (int m = 0; m < KM; ++m) {
        lv[m] = -INFINITY;
        li[m] = INT_MAX;
    }
    auto insert = [&](float v, int x) {
        bool c[KM];   // c[m]: (v, x) goes before entry m; monotone in m
#pragma unroll
        for (int m = 0; m < KM; ++m)
            c[m] = li[m] == INT_MAX || before(v, x, lv[m], li[m]);
#pragma unroll
        for (int m = KM - 1; m > 0; --m) {
            lv[m] = c[m - 1] ? lv[m - 1] : (c[m] ? v : lv[m]);
            li[m] = c[m - 1] ? li[m - 1] : (c[m] ? x : li[m]);
        }
        lv[0] = c[0] ? v : lv[0];
        li[0] = c[0] ? x : li[0];
    };
    if (vec) {   // float4 loads, kLoadBatch in flight per thread
        const float4 *p4 = reinterpret_cast<const float4 *>(p);
        const int n4 = V >> 2;
        int x4 = threadIdx.x;
        for (; x4 + (kLoadBatch - 1) * kExpandThreads < n4; x4 += kLoadBatch * kExpandThreads) {
            float4 t[kLoadBatch];
#pragma unroll
            for (int u = 0; u < kLoadBatch; ++u)
                t[u] = __ldg(p4 + x4 + u * kExpandThreads);
#pragma unroll
            for (int u = 0; u < kLoadBatch; ++u) {
                const int x = 4 * (x4 + u * kExpandThreads);
                insert(t[u].x, x);
                insert(t[u].y, x + 1);
                insert(t[u].z, x + 2);
                insert(t[u].w, x + 3);
            }
        }
        for (; x4 < n4; x4 += kExpandThreads) {
            const float4 t = __ldg(p4 + x4);
            insert(t.x, 4 * x4);
            insert(t.y, 4 * x4 + 1);
            insert(t.z, 4 * x4 + 2);
            insert(t.w, 4 * x4 + 3);
        }
    } else {
        for (int x = threadIdx.x; x < V; x += kExpandThreads)
            insert(__ldg(p + x), x);
    }
    for (int j = 0; j < k; ++j) {
        float bv = lv[0];
        int bi = li[0];
        block_best(bv, bi, shv, shi);
        if (li[0] == bi && bi != INT_MAX) {   // this thread's head won: pop it
#pragma unroll
            for (int m = 0; m < KM - 1; ++m) {
                lv[m] = lv[m + 1];
                li[m] = li[m + 1];
            }
            lv[KM - 1] = -INFINITY;
            li[KM - 1] = INT_MAX;
        }
        if (threadIdx.x == 0)
            emit(j, bi);
    }
}

__global__ void __launch_bounds__(kExpandThreads)
    tree_expand_kernel(const float *__restrict__ q_probs, int Rq, int V,
                       const int32_t *__restrict__ frow, int k, int32_t *__restrict__ parent,
                       int32_t *__restrict__ tokens, int32_t *__restrict__ q_row,
                       const int32_t *__restrict__ n_nodes, const int32_t *__restrict__ lvl_begin,
                       int Tmax)
{
    __shared__ float shv[kExpandThreads / 32];
    __shared__ int shi[kExpandThreads / 32];
    // sequence fastest: the working CTAs (i < F) of every sequence come first
    // in launch order, the idle ones after them
    const int b = blockIdx.x, i = blockIdx.y;
    // the frontier size from two loads; CTAs beyond it leave at once
    const int n = n_nodes[b], lb = lvl_begin[b];
    const int F = n == 0 ? 1 : n - lb;
    if (n < 0 || n > Tmax || k < 1 || k > V || F < 1 || lb < 0 ||
        (long)n + (long)F * k > Tmax || i >= F)
        return;
    // every q row of the frontier in range (the same answer in every CTA)
    int bad = 0;
    for (int f = threadIdx.x; f < F; f += kExpandThreads) {
        const int r = frow[(size_t)b * Tmax + f];
        bad |= r < 0 || r >= Rq;
    }
    if (__syncthreads_or(bad))
        return;
    const int r = frow[(size_t)b * Tmax + i];
    const float *p = q_probs + ((size_t)b * Rq + r) * V;
    const bool vec = (V & 3) == 0 && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
    auto emit = [&](int j, int tok) {
        if (in_bounds(n + i * k + j, Tmax, nullptr)) {
            const size_t u = (size_t)b * Tmax + n + i * k + j;
            parent[u] = n == 0 ? -1 : lb + i;
            tokens[u] = tok;   // k <= V: a pick always exists
            q_row[u] = r;
        }
    };
    // up to 8 children: one pass over the row; more: one pass per child
    if (k <= 2) {
        row_topk_one_pass<2>(p, V, vec, k, shv, shi, emit);
        return;
    }
    if (k <= 4) {
        row_topk_one_pass<4>(p, V, vec, k, shv, shi, emit);
        return;
    }
    if (k <= 8) {
        row_topk_one_pass<8>(p, V, vec, k, shv, shi, emit);
        return;
    }
    float pv = 0.f;
    int pi = -1;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = INT_MAX;
        auto consider = [&](float v, int x) {
            if (pi >= 0 && !before(pv, pi, v, x))
                return;   // at or before the previous pick
            if (bi == INT_MAX || before(v, x, bv, bi)) {
                bv = v;
                bi = x;
            }
        };
        if (vec) {   // float4 loads, kLoadBatch in flight per thread
            const float4 *p4 = reinterpret_cast<const float4 *>(p);
            const int n4 = V >> 2;
            int x4 = threadIdx.x;
            for (; x4 + (kLoadBatch - 1) * kExpandThreads < n4;
                 x4 += kLoadBatch * kExpandThreads) {
                float4 t[kLoadBatch];
#pragma unroll
                for (int u = 0; u < kLoadBatch; ++u)
                    t[u] = __ldg(p4 + x4 + u * kExpandThreads);
#pragma unroll
                for (int u = 0; u < kLoadBatch; ++u) {
                    const int x = 4 * (x4 + u * kExpandThreads);
                    consider(t[u].x, x);
                    consider(t[u].y, x + 1);
                    consider(t[u].z, x + 2);
                    consider(t[u].w, x + 3);
                }
            }
            for (; x4 < n4; x4 += kExpandThreads) {
                const float4 t = __ldg(p4 + x4);
                consider(t.x, 4 * x4);
                consider(t.y, 4 * x4 + 1);
                consider(t.z, 4 * x4 + 2);
                consider(t.w, 4 * x4 + 3);
            }
        } else {
            int x = threadIdx.x;
            for (; x + (kLoadBatch - 1) * kExpandThreads < V; x += kLoadBatch * kExpandThreads) {
                float t[kLoadBatch];
#pragma unroll
                for (int u = 0; u < kLoadBatch; ++u)
                    t[u] = __ldg(p + x + u * kExpandThreads);
#pragma unroll
                for (int u = 0; u < kLoadBatch; ++u)
                    consider(t[u], x + u * kExpandThreads);
            }
            for (; x < V; x += kExpandThreads)
                consider(__ldg(p + x), x);
        }
        block_best(bv, bi, shv, shi);
        pv = bv;
        pi = bi;
        if (threadIdx.x == 0)
            emit(j, pi);
    }
}

__global__ void tree_expand_commit_kernel(const int32_t *__restrict__ frow, int Rq, int V, int k,
                                          int32_t *__restrict__ n_nodes,
                                          int32_t *__restrict__ lvl_begin, int B, int Tmax,
                                          int32_t *dev_status)
{
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B)
        return;
    int n, lb;
    const int F = expand_frontier(frow, Rq, V, k, n_nodes, lvl_begin, b, Tmax, n, lb);
    if (F == 0) {
        flag(dev_status, TSD_DEV_BAD_TREE);
        return;
    }
    lvl_begin[b] = n;
    n_nodes[b] = n + F * k;
}

// Pre-order of the tree held in shared memory (par, first child, next
// sibling; -1 = none), written to order[]: returns the node count visited.
__device__ int preorder(const int *par, const int *fc, const int *ns, int root_first, int *order)
{
    int cnt = 0;
    int u = root_first;
    while (u >= 0) {
        order[cnt++] = u;
        if (fc[u] >= 0) {
            u = fc[u];
            continue;
        }
        while (u >= 0 && ns[u] < 0)
            u = par[u];
        if (u >= 0)
            u = ns[u];
    }
    return cnt;
}

__global__ void tree_dfs_kernel(const int32_t *__restrict__ parent,
                                const int32_t *__restrict__ tokens,
                                const int32_t *__restrict__ q_row,
                                const int32_t *__restrict__ n_nodes, int Tmax,
                                int32_t *__restrict__ perm, int32_t *__restrict__ out_parent,
                                int32_t *__restrict__ out_tokens, int32_t *__restrict__ out_q_row,
                                int32_t *dev_status)
{
    __shared__ int par[kMaxTree], fc[kMaxTree], ns[kMaxTree], order[kMaxTree], inv[kMaxTree];
    __shared__ int s_cnt;
    const int b = blockIdx.x, lane = threadIdx.x;   // one warp
    const int T = n_nodes[b];
    if (T < 0 || T > Tmax) {
        if (lane == 0)
            flag(dev_status, TSD_DEV_BAD_TREE);
        return;
    }
    bool bad = false;
    for (int v = lane; v < T; v += 32) {   // the loads in parallel
        par[v] = parent[(size_t)b * Tmax + v];
        bad |= par[v] < -1 || par[v] >= v;
    }
    if (__any_sync(0xffffffffu, bad)) {
        if (lane == 0)
            flag(dev_status, TSD_DEV_BAD_TREE);
        return;
    }
    __syncwarp();
    if (lane == 0) {   // the walk, on shared memory
        int root_first = -1;
        for (int v = T - 1; v >= 0; --v)   // children lists in increasing index
            fc[v] = -1;
        for (int v = T - 1; v >= 0; --v) {
            const int p = par[v];
            if (p < 0) {
                ns[v] = root_first;
                root_first = v;
            } else {
                ns[v] = fc[p];
                fc[p] = v;
            }
        }
        s_cnt = preorder(par, fc, ns, root_first, order);
        for (int i = 0; i < s_cnt; ++i)
            inv[order[i]] = i;
    }
    __syncwarp();
    for (int i = lane; i < s_cnt; i += 32) {
        const int u = order[i];
        if (!in_bounds(i, Tmax, nullptr) || !in_bounds(u, Tmax, nullptr))
            continue;
        const size_t o = (size_t)b * Tmax + i;
        perm[o] = u;
        out_parent[o] = par[u] < 0 ? -1 : inv[par[u]];
        out_tokens[o] = tokens[(size_t)b * Tmax + u];
        out_q_row[o] = q_row[(size_t)b * Tmax + u];
    }
}

__global__ void tree_merge_kernel(const int32_t *__restrict__ ctok, const int32_t *__restrict__ cq,
                                  const int32_t *__restrict__ clen, int M, int L, int Tmax,
                                  int32_t *__restrict__ parent, int32_t *__restrict__ tokens,
                                  int32_t *__restrict__ q_row, int32_t *__restrict__ n_nodes,
                                  int32_t *dev_status)
{
    __shared__ int par[kMaxTree], tok[kMaxTree], qr[kMaxTree], fc[kMaxTree], lc[kMaxTree],
        ns[kMaxTree], order[kMaxTree], inv[kMaxTree];
    __shared__ int s_ct[kMergeStage], s_cq[kMergeStage], s_len[kMergeStage];
    const int b = blockIdx.x, lane = threadIdx.x;   // one warp
    // the chains into shared memory in parallel when they fit
    const bool staged = M * L <= kMergeStage;
    if (staged) {
        for (int i = lane; i < M * L; i += 32) {
            s_ct[i] = ctok[(size_t)b * M * L + i];
            s_cq[i] = cq[(size_t)b * M * L + i];
        }
        for (int m = lane; m < M; m += 32)
            s_len[m] = clen[(size_t)b * M + m];
    }
    __syncwarp();
    if (lane != 0)
        return;
    const int *ct = staged ? s_ct : ctok + (size_t)b * M * L;
    const int *cqr = staged ? s_cq : cq + (size_t)b * M * L;
    const int *cl = staged ? s_len : clen + (size_t)b * M;
    int T = 0, root_first = -1, root_last = -1;
    bool ok = true;
    for (int m = 0; ok && m < M; ++m) {
        const int len = cl[m];
        if (len < 0 || len > L) {
            ok = false;
            break;
        }
        int cur = -1;
        for (int i = 0; i < len; ++i) {
            const int t = ct[(size_t)m * L + i];
            int v = cur < 0 ? root_first : fc[cur];
            while (v >= 0 && tok[v] != t)
                v = ns[v];
            if (v < 0) {   // a new node, last child of cur
                if (T == Tmax) {
                    ok = false;
                    break;
                }
                v = T++;
                par[v] = cur;
                tok[v] = t;
                qr[v] = cqr[(size_t)m * L + i];
                fc[v] = lc[v] = ns[v] = -1;
                if (cur < 0) {
                    if (root_last < 0)
                        root_first = v;
                    else
                        ns[root_last] = v;
                    root_last = v;
                } else {
                    if (lc[cur] < 0)
                        fc[cur] = v;
                    else
                        ns[lc[cur]] = v;
                    lc[cur] = v;
                }
            }
            cur = v;
        }
    }
    if (!ok) {
        n_nodes[b] = -1;
        flag(dev_status, TSD_DEV_BAD_TREE);
        return;
    }
    const int cnt = preorder(par, fc, ns, root_first, order);
    for (int i = 0; i < cnt; ++i)
        inv[order[i]] = i;
    for (int i = 0; i < cnt; ++i) {
        const int u = order[i];
        if (!in_bounds(i, Tmax, dev_status))
            break;
        const size_t o = (size_t)b * Tmax + i;
        parent[o] = par[u] < 0 ? -1 : inv[par[u]];
        tokens[o] = tok[u];
        q_row[o] = qr[u];
    }
    n_nodes[b] = cnt;
}

}  // namespace

int launch_tree_expand(const float *q_probs, int Rq, int V, const int32_t *frow, int k,
                       int32_t *parent, int32_t *tokens, int32_t *q_row, int32_t *n_nodes,
                       int32_t *lvl_begin, int B, int Tmax, int32_t *dev_status,
                       cudaStream_t stream)
{
    if (B == 0)
        return TSD_OK;
    tree_expand_kernel<<<dim3(B, Tmax), kExpandThreads, 0, stream>>>(
        q_probs, Rq, V, frow, k, parent, tokens, q_row, n_nodes, lvl_begin, Tmax);
    TSD_LAUNCH_CHECK();
    tree_expand_commit_kernel<<<(B + 127) / 128, 128, 0, stream>>>(frow, Rq, V, k, n_nodes,
                                                                  lvl_begin, B, Tmax, dev_status);
    TSD_LAUNCH_CHECK();
    return TSD_OK;
}

int launch_tree_dfs(const int32_t *parent, const int32_t *tokens, const int32_t *q_row,
                    const int32_t *n_nodes, int B, int Tmax, int32_t *perm, int32_t *out_parent,
                    int32_t *out_tokens, int32_t *out_q_row, int32_t *dev_status,
                    cudaStream_t stream)
{
    if (B == 0)
        return TSD_OK;
    tree_dfs_kernel<<<B, 32, 0, stream>>>(parent, tokens, q_row, n_nodes, Tmax, perm, out_parent,
                                          out_tokens, out_q_row, dev_status);
    TSD_LAUNCH_CHECK();
    return TSD_OK;
}

int launch_tree_merge(const int32_t *ctok, const int32_t *cq, const int32_t *clen, int M, int L,
                      int B, int Tmax, int32_t *parent, int32_t *tokens, int32_t *q_row,
                      int32_t *n_nodes, int32_t *dev_status, cudaStream_t stream)
{
    if (B == 0)
        return TSD_OK;
    tree_merge_kernel<<<B, 32, 0, stream>>>(ctok, cq, clen, M, L, Tmax, parent, tokens, q_row,
                                            n_nodes, dev_status);
    TSD_LAUNCH_CHECK();
    return TSD_OK;
}

}  // namespace tsd
