/*
 * CPU oracle for SpecInfer-style tree verification -- TEST INFRASTRUCTURE.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load this library.  It shares no code, header, table or helper with the
 * CUDA library; the two only see the same seeded inputs.
 *
 * Everything is computed in fp64 from the exact input values, in the plain
 * order of the definitions on the page "論文解説: SpecInfer - 投機的推論と
 * トークンツリー検証によるLLMサービング高速化" (0h-n0.github.io):
 *
 *   - S_u and tree attention:  section "トークンツリー構造の仕組み", the
 *     definition of S_u and the Attention(Q_u, K_{S_u}, V_{S_u}) equation.
 *   - topology-aware mask:     same section (a node attends only to its
 *     ancestors) and "Tree Attention のカーネル融合", item 1.
 *   - greedy verification:     "ツリー検証アルゴリズム" (greedy variant) and the
 *     "accept the matching prefix plus one target token" rule of the
 *     flatkey.ai speculative decoding guide (its verification diagram).
 *   - stochastic verification: "ツリー検証アルゴリズム", the P_accept equation
 *     min(1, P_LLM/P_SSM) and the residual equation norm(max(0, P_LLM-P_SSM)).
 *   - committing the accepted path: "Tree Attention のカーネル融合", item 2
 *     (the tree's KV entries stay consistent with the existing KV cache),
 *     and the flatkey.ai guide's verification diagram (the accepted prefix
 *     is committed).
 *
 * Readings taken where the page is silent:
 *   - the committed prefix is always attended; S_u = prefix, then the tree
 *     path root-first, ending with u itself;
 *   - the root is the last committed token (logits row 0); node u owns
 *     logits row 1+u; parent[u] = -1 marks a child of the root;
 *   - siblings are tried in ascending node index; after a rejected sibling
 *     the target distribution becomes norm(max(0, p - q_sibling)) before the
 *     next sibling is tried; if the residual sums to 0 it stays unchanged;
 *   - acceptance uses the division-free form u*q(x) <= p(x) with p(x) > 0;
 *   - a draw takes the smallest token i whose cumulative sum C_i > u (C in
 *     ascending token order); if rounding leaves none, the largest i with
 *     p_i > 0;
 *   - a node that accepts none of its children (or has none) ends the
 *     sequence with a draw at its own row using u_sample[row];
 *   - greedy: the longest root path all of whose tokens equal the argmax of
 *     their parent's row (lowest token id on argmax ties, lowest terminal
 *     node index on length ties), then the argmax of the terminal's row;
 *   - commit: the accepted nodes' K and V rows move to the positions right
 *     after the prefix, in path order, and the prefix grows by their number
 *     (the final sampled token has no KV entry yet).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BAD_TREE 1
#define ORACLE_BAD_TOKEN 2
#define ORACLE_BAD_QROW 4
#define ORACLE_BAD_PATH 32

/* dtype 0: IEEE fp32, dtype 1: bfloat16 (upper 16 bits of an fp32). */
static double load_value(const void *base, size_t i, int dtype)
{
    if (dtype == 0)
        return (double)((const float *)base)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* A tree of T nodes is well formed iff every parent precedes its child. */
static int tree_is_valid(const int32_t *parent, int T)
{
    for (int u = 0; u < T; ++u)
        if (parent[u] < -1 || parent[u] >= u)
            return 0;
    return 1;
}

/* Root-first path of node u: writes the nodes and returns their count. */
static int root_path(const int32_t *parent, int u, int32_t *path)
{
    int n = 0;
    for (int v = u; v >= 0; v = parent[v])
        path[n++] = v;
    for (int i = 0; i < n / 2; ++i) {
        int32_t t = path[i];
        path[i] = path[n - 1 - i];
        path[n - 1 - i] = t;
    }
    return n;
}

/*
 * Ancestor-or-self mask: bit v of mask[b][u] is set iff node v lies on the
 * path root -> u (u included).  depth[b][u] = number of nodes on that path.
 * first_child[b][1+c] / first_child[b][0] (root) = smallest child index or -1;
 * next_sibling[b][u] = next larger node index with the same parent, or -1.
 * Padding slots (u >= n_nodes[b]) get mask 0, depth 0 and -1 links.
 */
int oracle_tree_mask(const int32_t *parent, const int32_t *n_nodes, int B, int Tmax,
                     uint32_t *mask, int32_t *depth, int32_t *first_child,
                     int32_t *next_sibling, int32_t *status)
{
    int W = (Tmax + 31) / 32, any = 0;
    for (int b = 0; b < B; ++b) {
        const int32_t *par = parent + (size_t)b * Tmax;
        uint32_t *mk = mask + (size_t)b * Tmax * W;
        int32_t *dp = depth + (size_t)b * Tmax;
        int32_t *fc = first_child + (size_t)b * (Tmax + 1);
        int32_t *ns = next_sibling + (size_t)b * Tmax;
        memset(mk, 0, sizeof(uint32_t) * (size_t)Tmax * W);
        for (int u = 0; u < Tmax; ++u) {
            dp[u] = 0;
            ns[u] = -1;
        }
        for (int s = 0; s <= Tmax; ++s)
            fc[s] = -1;
        status[b] = 0;
        int T = n_nodes[b];
        if (T < 0 || T > Tmax || !tree_is_valid(par, T)) {
            status[b] = ORACLE_BAD_TREE;
            any |= ORACLE_BAD_TREE;
            continue;
        }
        for (int u = 0; u < T; ++u) {
            int d = 0;
            for (int v = u; v >= 0; v = par[v]) {
                mk[(size_t)u * W + v / 32] |= 1u << (v % 32);
                ++d;
            }
            dp[u] = d;
        }
        for (int u = 0; u < T; ++u) {
            if (fc[par[u] + 1] < 0)
                fc[par[u] + 1] = u;
            for (int v = u + 1; v < T; ++v)
                if (par[v] == par[u]) {
                    ns[u] = v;
                    break;
                }
        }
    }
    return any;
}

/*
 * Attention of one query row (b, u, h):
 *   o = sum_{j in S_u} softmax_j(scale * q . k_j) v_j,
 * S_u = prefix positions 0..P_b-1 followed by the cache positions P_b + v of
 * the nodes v on the root -> u path (root-first, u last).  GQA: query head h
 * reads KV head h / (Hq / Hkv).  q is [B][Tmax][Hq][D]; k, v are
 * [B][Hkv][Lmax][D].  `work` holds Tmax int32 + (Lmax) doubles.
 */
static void attention_row(const void *q, const void *k, const void *v, int dtype,
                          const int32_t *prefix_len, const int32_t *parent, int b, int u,
                          int h, int Tmax, int Hq, int Hkv, int D, int Lmax, double scale,
                          int32_t *path, double *score, double *out)
{
    int G = Hq / Hkv, hk = h / G;
    int P = prefix_len[b];
    int np = root_path(parent + (size_t)b * Tmax, u, path);
    int n = P + np;
    size_t qoff = (((size_t)b * Tmax + u) * Hq + h) * D;
    size_t kvbase = ((size_t)b * Hkv + hk) * (size_t)Lmax;
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        int pos = j < P ? j : P + path[j - P];
        size_t koff = (kvbase + pos) * D;
        double s = 0.0;
        for (int d = 0; d < D; ++d)
            s += load_value(q, qoff + d, dtype) * load_value(k, koff + d, dtype);
        s *= scale;
        score[j] = s;
        if (s > m)
            m = s;
    }
    double Z = 0.0;
    for (int j = 0; j < n; ++j) {
        score[j] = exp(score[j] - m);
        Z += score[j];
    }
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    for (int j = 0; j < n; ++j) {
        int pos = j < P ? j : P + path[j - P];
        size_t voff = (kvbase + pos) * D;
        double w = score[j] / Z;
        for (int d = 0; d < D; ++d)
            out[d] += w * load_value(v, voff + d, dtype);
    }
}

/* Every row (b, u < n_nodes[b], h) into out[B][Tmax][Hq][D]; padding rows
 * are left untouched.  Returns ORACLE_BAD_TREE if a tree is malformed (its
 * rows are then skipped). */
int oracle_tree_attention(const void *q, const void *k, const void *v, int dtype,
                          const int32_t *prefix_len, const int32_t *n_nodes,
                          const int32_t *parent, int B, int Tmax, int Hq, int Hkv, int D,
                          int Lmax, double scale, double *out)
{
    int bad = 0;
    for (int b = 0; b < B; ++b)
        if (n_nodes[b] < 0 || n_nodes[b] > Tmax ||
            !tree_is_valid(parent + (size_t)b * Tmax, n_nodes[b]) ||
            prefix_len[b] < 0 || prefix_len[b] + n_nodes[b] > Lmax)
            bad = ORACLE_BAD_TREE;
    if (bad)
        return bad;
    long total = (long)B * Tmax * Hq;
#pragma omp parallel
    {
        int32_t *path = (int32_t *)malloc(sizeof(int32_t) * (size_t)(Tmax + 1));
        double *score = (double *)malloc(sizeof(double) * (size_t)(Lmax + 1));
#pragma omp for schedule(dynamic, 4)
        for (long i = 0; i < total; ++i) {
            int h = (int)(i % Hq);
            int u = (int)((i / Hq) % Tmax);
            int b = (int)(i / ((long)Hq * Tmax));
            if (u >= n_nodes[b])
                continue;
            attention_row(q, k, v, dtype, prefix_len, parent, b, u, h, Tmax, Hq, Hkv, D, Lmax,
                          scale, path, score, out + (size_t)i * D);
        }
        free(path);
        free(score);
    }
    return 0;
}

/* Selected rows: sel[3*i .. 3*i+2] = (b, u, h); out is [nsel][D]. */
int oracle_tree_attention_rows(const void *q, const void *k, const void *v, int dtype,
                               const int32_t *prefix_len, const int32_t *n_nodes,
                               const int32_t *parent, int B, int Tmax, int Hq, int Hkv, int D,
                               int Lmax, double scale, int nsel, const int32_t *sel,
                               double *out)
{
    for (int i = 0; i < nsel; ++i) {
        int b = sel[3 * i], u = sel[3 * i + 1];
        if (b < 0 || b >= B || u < 0 || u >= n_nodes[b] ||
            !tree_is_valid(parent + (size_t)b * Tmax, n_nodes[b]))
            return ORACLE_BAD_TREE;
    }
#pragma omp parallel
    {
        int32_t *path = (int32_t *)malloc(sizeof(int32_t) * (size_t)(Tmax + 1));
        double *score = (double *)malloc(sizeof(double) * (size_t)(Lmax + 1));
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < nsel; ++i)
            attention_row(q, k, v, dtype, prefix_len, parent, sel[3 * i], sel[3 * i + 1],
                          sel[3 * i + 2], Tmax, Hq, Hkv, D, Lmax, scale, path, score,
                          out + (size_t)i * D);
        free(path);
        free(score);
    }
    return 0;
}

/* Checks shared by both verifiers; returns a status bit set. */
static int check_sequence(const int32_t *par, const int32_t *tok, const int32_t *qrow, int T,
                          int Tmax, int V, int Rq)
{
    if (T < 0 || T > Tmax || !tree_is_valid(par, T))
        return ORACLE_BAD_TREE;
    for (int u = 0; u < T; ++u)
        if (tok[u] < 0 || tok[u] >= V)
            return ORACLE_BAD_TOKEN;
    if (qrow)
        for (int u = 0; u < T; ++u)
            if (qrow[u] < 0 || qrow[u] >= Rq)
                return ORACLE_BAD_QROW;
    return 0;
}

/* Lowest index among the maxima of a row. */
static int row_argmax(const float *l, int V)
{
    int best = 0;
    for (int i = 1; i < V; ++i)
        if (l[i] > l[best])
            best = i;
    return best;
}

/*
 * Greedy verification.  logits [B][Tmax+1][V] (row 0 = root, row 1+u = node u).
 * Outputs: out_path[b][0..n-1] = accepted nodes (root-first),
 * out_tokens[b][0..n] = their tokens followed by the argmax of the last
 * accepted node's row (row 0 if none), n_accepted[b] = n.  Other entries are
 * not written.  A malformed sequence gets n_accepted = -1 and a status bit.
 */
int oracle_verify_greedy(const float *logits, const int32_t *tokens, const int32_t *parent,
                         const int32_t *n_nodes, int B, int Tmax, int V, int32_t *out_tokens,
                         int32_t *out_path, int32_t *n_accepted, int32_t *status)
{
    int any = 0;
    for (int b = 0; b < B; ++b) {
        const int32_t *par = parent + (size_t)b * Tmax;
        const int32_t *tok = tokens + (size_t)b * Tmax;
        int T = n_nodes[b];
        status[b] = check_sequence(par, tok, NULL, T, Tmax, V, 0);
        if (status[b]) {
            any |= status[b];
            n_accepted[b] = -1;
            continue;
        }
        const float *L = logits + (size_t)b * (Tmax + 1) * V;
        int32_t *matched = (int32_t *)calloc((size_t)T + 1, sizeof(int32_t));
        int32_t *len = (int32_t *)calloc((size_t)T + 1, sizeof(int32_t));
        int best = -1, best_len = 0;
        for (int u = 0; u < T; ++u) {
            int p = par[u];
            int parent_ok = p < 0 ? 1 : matched[p];
            matched[u] = parent_ok && tok[u] == row_argmax(L + (size_t)(p + 1) * V, V);
            len[u] = (p < 0 ? 0 : len[p]) + 1;
            if (matched[u] && len[u] > best_len) {
                best = u;
                best_len = len[u];
            }
        }
        int32_t *path = out_path + (size_t)b * Tmax;
        int32_t *otk = out_tokens + (size_t)b * (Tmax + 1);
        int n = best >= 0 ? root_path(par, best, path) : 0;
        for (int i = 0; i < n; ++i)
            otk[i] = tok[path[i]];
        otk[n] = row_argmax(L + (size_t)(best + 1) * V, V);
        n_accepted[b] = n;
        free(matched);
        free(len);
    }
    return any;
}

/*
 * Stochastic verification by multi-step speculative sampling, walking the
 * tree from the root as the page's verify procedure does:
 *   p = softmax(l_row / T) for the current node's row;
 *   for each child c (ascending index) with token x and SSM row q_c:
 *       accept iff p(x) > 0 and u_accept[c] * q_c(x) <= p(x);
 *       on accept: emit x, move to c, restart with c's row;
 *       on reject: p <- max(0, p - q_c) / sum(max(0, p - q_c));
 *   if no child is accepted: emit the inverse-CDF draw of p at u_sample[row].
 * Boundary diagnostics: a decision is flagged when |u*q(x) - p(x)| <= 1e-9*q(x)
 * (acceptance) or |u - C_i| <= 1e-9 for some cumulative sum C_i (draw).
 * n_flagged[b] / n_decisions[b] count them along the path.
 */
int oracle_verify_stochastic(const float *logits, double temperature, const float *qprobs,
                             const int32_t *q_row, int Rq, const int32_t *tokens,
                             const int32_t *parent, const int32_t *n_nodes,
                             const double *u_accept, const double *u_sample, int B, int Tmax,
                             int V, int32_t *out_tokens, int32_t *out_path,
                             int32_t *n_accepted, int32_t *n_flagged, int32_t *n_decisions,
                             int32_t *status)
{
    int any = 0;
    for (int b = 0; b < B; ++b) {
        const int32_t *par = parent + (size_t)b * Tmax;
        const int32_t *tok = tokens + (size_t)b * Tmax;
        const int32_t *qr = q_row + (size_t)b * Tmax;
        int T = n_nodes[b];
        status[b] = check_sequence(par, tok, qr, T, Tmax, V, Rq);
        n_flagged[b] = 0;
        n_decisions[b] = 0;
        if (status[b]) {
            any |= status[b];
            n_accepted[b] = -1;
        }
    }
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)V);
#pragma omp for schedule(dynamic, 1)
        for (int b = 0; b < B; ++b) {
            if (status[b])
                continue;
            const int32_t *par = parent + (size_t)b * Tmax;
            const int32_t *tok = tokens + (size_t)b * Tmax;
            const int32_t *qr = q_row + (size_t)b * Tmax;
            const float *L = logits + (size_t)b * (Tmax + 1) * V;
            const float *Q = qprobs + (size_t)b * Rq * V;
            int32_t *path = out_path + (size_t)b * Tmax;
            int32_t *otk = out_tokens + (size_t)b * (Tmax + 1);
            int T = n_nodes[b], n = 0, flagged = 0, decisions = 0;
            int cur = -1;
            for (;;) {
                int row = cur + 1;
                const float *l = L + (size_t)row * V;
                double m = -INFINITY;
                for (int i = 0; i < V; ++i)
                    if ((double)l[i] > m)
                        m = (double)l[i];
                double Z = 0.0;
                for (int i = 0; i < V; ++i)
                    Z += exp(((double)l[i] - m) / temperature);
                for (int i = 0; i < V; ++i)
                    p[i] = exp(((double)l[i] - m) / temperature) / Z;
                int accepted = -1;
                for (int c = 0; c < T; ++c) {
                    if (par[c] != cur)
                        continue;
                    const float *qc = Q + (size_t)qr[c] * V;
                    int x = tok[c];
                    double qx = (double)qc[x], px = p[x], u = u_accept[(size_t)b * Tmax + c];
                    ++decisions;
                    if (fabs(u * qx - px) <= 1e-9 * qx)
                        ++flagged;
                    if (px > 0.0 && u * qx <= px) {
                        accepted = c;
                        break;
                    }
                    double S = 0.0;
                    for (int i = 0; i < V; ++i) {
                        double r = p[i] - (double)qc[i];
                        S += r > 0.0 ? r : 0.0;
                    }
                    if (S > 0.0)
                        for (int i = 0; i < V; ++i) {
                            double r = p[i] - (double)qc[i];
                            p[i] = (r > 0.0 ? r : 0.0) / S;
                        }
                }
                if (accepted >= 0) {
                    path[n] = accepted;
                    otk[n] = tok[accepted];
                    ++n;
                    cur = accepted;
                    continue;
                }
                double u = u_sample[(size_t)b * (Tmax + 1) + row], C = 0.0;
                int pick = -1, near = 0;
                for (int i = 0; i < V; ++i) {
                    C += p[i];
                    if (fabs(u - C) <= 1e-9)
                        near = 1;
                    if (pick < 0 && C > u)
                        pick = i;
                }
                if (pick < 0)
                    for (int i = V - 1; i >= 0; --i)
                        if (p[i] > 0.0) {
                            pick = i;
                            break;
                        }
                ++decisions;
                flagged += near;
                otk[n] = pick;
                break;
            }
            n_accepted[b] = n;
            n_flagged[b] = flagged;
            n_decisions[b] = decisions;
        }
        free(p);
    }
    return any;
}

/* Commit of the accepted path.  For each sequence b with n = n_accepted[b]
 * >= 0 and path u_0..u_{n-1} = out_path[b][0..n-1]: for every KV head, the
 * K row and the V row at cache position P_b + u_i move to P_b + i, all at
 * once (every source is read before any destination is written), and
 * new_prefix[b] = P_b + n.  Rows are moved as raw bytes.  Sequences with
 * n < 0 are left alone (new_prefix = P_b).  A path that is not a strictly
 * increasing list of node indices in [0, Tmax), longer than Tmax, or that
 * reaches past Lmax, sets status[b] = ORACLE_BAD_PATH and moves nothing. */
int oracle_kv_commit(unsigned char *k, unsigned char *v, const int32_t *prefix_len,
                     const int32_t *out_path, const int32_t *n_accepted, int B, int Tmax, int Hkv,
                     int Lmax, int row_bytes, int32_t *new_prefix, int32_t *status)
{
    int any = 0;
    unsigned char *tmp = (unsigned char *)malloc((size_t)(Tmax > 0 ? Tmax : 1) * row_bytes);
    for (int b = 0; b < B; ++b) {
        const int n = n_accepted[b], P = prefix_len[b];
        const int32_t *path = out_path + (size_t)b * Tmax;
        new_prefix[b] = P;
        status[b] = 0;
        if (n < 0)
            continue;
        int ok = n <= Tmax && P >= 0;
        for (int i = 0; ok && i < n; ++i) {
            const int u = path[i];
            if (u < 0 || u >= Tmax || (i > 0 && u <= path[i - 1]) || P + u >= Lmax)
                ok = 0;
        }
        if (!ok) {
            status[b] = ORACLE_BAD_PATH;
            any |= ORACLE_BAD_PATH;
            continue;
        }
        for (int h = 0; h < Hkv; ++h) {
            unsigned char *planes[2] = {k, v};
            for (int t = 0; t < 2; ++t) {
                unsigned char *base = planes[t] + ((size_t)b * Hkv + h) * Lmax * row_bytes;
                for (int i = 0; i < n; ++i)
                    memcpy(tmp + (size_t)i * row_bytes,
                           base + (size_t)(P + path[i]) * row_bytes, row_bytes);
                for (int i = 0; i < n; ++i)
                    memcpy(base + (size_t)(P + i) * row_bytes, tmp + (size_t)i * row_bytes,
                           row_bytes);
            }
        }
        new_prefix[b] = P + n;
    }
    free(tmp);
    return any;
}

/* ---------------------------------------------------------------- tree construction
 * Section "マルチドラフトモデルアプローチ" of the SpecInfer explainer: an
 * expansion-based tree <k_1, ..., k_n> takes the top-k_i tokens of one SSM at
 * every node of depth i-1 (item 1); a merge-based tree merges the outputs of
 * several SSMs into one token tree (item 2); "Tree Attention のカーネル融合",
 * item 2: the tree is laid out in depth-first order. */

/* (v, i) comes before (w, j) in "descending probability, lower token first". */
static int before(float v, int i, float w, int j) { return v > w || (v == w && i < j); }

/* One expansion level.  The frontier is the root (lvl_begin[b] == n_nodes[b]
 * == 0 only for an empty tree) or the nodes lvl_begin[b] .. n_nodes[b]-1;
 * frontier node i (in index order) has its SSM distribution in q row
 * frow[b][i].  Each frontier node gets k children, appended in frontier order,
 * holding the k best tokens of its row in descending probability (lower
 * token id on ties), with q_row = frow[b][i].  lvl_begin[b] becomes the old
 * n_nodes[b].  More than Tmax nodes, a bad q row or k > V: status 1, nothing
 * changes. */
int oracle_tree_expand(const float *q_probs, int Rq, int V, const int32_t *frow, int k,
                       int32_t *parent, int32_t *tokens, int32_t *q_row, int32_t *n_nodes,
                       int32_t *lvl_begin, int B, int Tmax, int32_t *status)
{
    int any = 0;
    for (int b = 0; b < B; ++b) {
        const int n = n_nodes[b];
        const int root_level = (n == 0);
        const int F = root_level ? 1 : n - lvl_begin[b];
        const int32_t *fr = frow + (size_t)b * Tmax;
        int ok = k >= 1 && k <= V && F >= 1 && lvl_begin[b] >= 0 && n + F * k <= Tmax;
        for (int i = 0; ok && i < F; ++i)
            ok = fr[i] >= 0 && fr[i] < Rq;
        status[b] = ok ? 0 : 1;
        if (!ok) {
            any |= 1;
            continue;
        }
        for (int i = 0; i < F; ++i) {
            const float *p = q_probs + ((size_t)b * Rq + fr[i]) * V;
            float pv = 0.f;
            int pi = -1;   /* the previous pick; the next is the best after it */
            for (int j = 0; j < k; ++j) {
                int best = -1;
                for (int x = 0; x < V; ++x) {
                    if (pi >= 0 && !before(pv, pi, p[x], x))
                        continue;
                    if (best < 0 || before(p[x], x, p[best], best))
                        best = x;
                }
                const int u = n + i * k + j;
                parent[(size_t)b * Tmax + u] = root_level ? -1 : lvl_begin[b] + i;
                tokens[(size_t)b * Tmax + u] = best;
                q_row[(size_t)b * Tmax + u] = fr[i];
                pv = p[best];
                pi = best;
            }
        }
        lvl_begin[b] = n;
        n_nodes[b] = n + F * k;
    }
    return any;
}

/* Depth-first pre-order of a tree given in any topological order (children
 * visited in increasing index): perm[new] = old, and parent/tokens/q_row
 * renumbered (out_*).  status 1 for a tree that is not topological. */
int oracle_tree_dfs_order(const int32_t *parent, const int32_t *tokens, const int32_t *q_row,
                          const int32_t *n_nodes, int B, int Tmax, int32_t *perm,
                          int32_t *out_parent, int32_t *out_tokens, int32_t *out_q_row,
                          int32_t *status)
{
    int any = 0;
    int32_t *stack = (int32_t *)malloc(sizeof(int32_t) * (Tmax + 1));
    int32_t *inv = (int32_t *)malloc(sizeof(int32_t) * (Tmax + 1));
    for (int b = 0; b < B; ++b) {
        const int T = n_nodes[b];
        const int32_t *par = parent + (size_t)b * Tmax;
        status[b] = (T < 0 || T > Tmax || !tree_is_valid(par, T)) ? 1 : 0;
        if (status[b]) {
            any |= 1;
            continue;
        }
        int top = 0, cnt = 0;
        /* push the root's children in decreasing index so the smallest pops first */
        for (int v = T - 1; v >= 0; --v)
            if (par[v] == -1)
                stack[top++] = v;
        while (top > 0) {
            const int u = stack[--top];
            perm[(size_t)b * Tmax + cnt] = u;
            inv[u] = cnt++;
            for (int v = T - 1; v > u; --v)
                if (par[v] == u)
                    stack[top++] = v;
        }
        for (int i = 0; i < T; ++i) {
            const int u = perm[(size_t)b * Tmax + i];
            out_parent[(size_t)b * Tmax + i] = par[u] < 0 ? -1 : inv[par[u]];
            out_tokens[(size_t)b * Tmax + i] = tokens[(size_t)b * Tmax + u];
            out_q_row[(size_t)b * Tmax + i] = q_row[(size_t)b * Tmax + u];
        }
    }
    free(stack);
    free(inv);
    return any;
}

/* Merge M chains per sequence into one token tree: chain m proposes tokens
 * ctok[b][m][0..clen[b][m]-1], step i drawn from q row cq[b][m][i].  A chain
 * reuses the node of an earlier chain while its prefix matches (same parent,
 * same token) and creates new nodes from the first difference on; a node
 * keeps the q row of the chain that created it.  Output in depth-first
 * pre-order, children in creation order.  More than Tmax nodes or a bad
 * length: status 1, n_nodes = -1. */
int oracle_tree_merge_chains(const int32_t *ctok, const int32_t *cq, const int32_t *clen, int M,
                             int L, int B, int Tmax, int32_t *parent, int32_t *tokens,
                             int32_t *q_row, int32_t *n_nodes, int32_t *status)
{
    int any = 0;
    int32_t *tp = (int32_t *)malloc(sizeof(int32_t) * (Tmax + 1));
    int32_t *tt = (int32_t *)malloc(sizeof(int32_t) * (Tmax + 1));
    int32_t *tq = (int32_t *)malloc(sizeof(int32_t) * (Tmax + 1));
    int32_t *perm = (int32_t *)malloc(sizeof(int32_t) * (Tmax + 1));
    int32_t *op = (int32_t *)malloc(sizeof(int32_t) * (Tmax + 1));
    int32_t *ot = (int32_t *)malloc(sizeof(int32_t) * (Tmax + 1));
    int32_t *oq = (int32_t *)malloc(sizeof(int32_t) * (Tmax + 1));
    for (int b = 0; b < B; ++b) {
        int T = 0, ok = 1;
        for (int m = 0; ok && m < M; ++m) {
            const int len = clen[(size_t)b * M + m];
            if (len < 0 || len > L) {
                ok = 0;
                break;
            }
            int cur = -1;
            for (int i = 0; i < len; ++i) {
                const int t = ctok[((size_t)b * M + m) * L + i];
                int found = -1;
                for (int v = 0; v < T; ++v)
                    if (tp[v] == cur && tt[v] == t) {
                        found = v;
                        break;
                    }
                if (found < 0) {
                    if (T == Tmax) {
                        ok = 0;
                        break;
                    }
                    tp[T] = cur;
                    tt[T] = t;
                    tq[T] = cq[((size_t)b * M + m) * L + i];
                    found = T++;
                }
                cur = found;
            }
        }
        status[b] = ok ? 0 : 1;
        if (!ok) {
            any |= 1;
            n_nodes[b] = -1;
            continue;
        }
        int32_t st;
        oracle_tree_dfs_order(tp, tt, tq, &T, 1, Tmax > 0 ? Tmax : 1, perm, op, ot, oq, &st);
        for (int u = 0; u < T; ++u) {
            parent[(size_t)b * Tmax + u] = op[u];
            tokens[(size_t)b * Tmax + u] = ot[u];
            q_row[(size_t)b * Tmax + u] = oq[u];
        }
        n_nodes[b] = T;
    }
    free(tp); free(tt); free(tq); free(perm); free(op); free(ot); free(oq);
    return any;
}
