/*
 * tsd.h -- C ABI of the B200 (sm_100a) tree speculative decoding verification
 * library (libtsd.so).
 *
 * The operations follow the SpecInfer explainer page "論文解説: SpecInfer -
 * 投機的推論とトークンツリー検証によるLLMサービング高速化" (0h-n0.github.io,
 * arXiv:2305.09781):
 *   - a token tree of speculated tokens, one node per token, each root-to-node
 *     path a candidate sequence S_u  (section "トークンツリー構造の仕組み");
 *   - topology-aware tree attention, softmax(Q_u K_{S_u}^T / sqrt(d_k)) V_{S_u},
 *     where a node sees only its ancestors (same section, and "Tree Attention
 *     のカーネル融合", item 1);
 *   - greedy and stochastic (multi-step speculative sampling) verification of
 *     the tree from the target model's logits (section "ツリー検証アルゴリズム").
 *
 * Common conventions
 * ------------------
 *  - Every pointer is a DEVICE pointer owned by the caller unless stated
 *    otherwise; tensors are dense and row-major in the stated shape.  The
 *    library never allocates device memory: scratch comes from a caller
 *    workspace whose size the matching *_workspace_size() call returns.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and never synchronizes.  Calls are reentrant across
 *    streams; a workspace must not be shared by calls that may overlap.
 *  - A tree has n_nodes[b] = T_b <= Tmax nodes (Tmax <= TSD_MAX_TREE).  Node u
 *    has parent[b][u] in [-1, u-1]; -1 means "child of the root".  The root is
 *    the last committed token: it is part of the prefix, not a tree node.
 *    Slots u >= T_b are padding; outputs for them are not written unless a
 *    function says so.
 *  - The KV cache is [B][Hkv][Lmax][D]: the committed prefix of sequence b at
 *    positions 0..prefix_len[b]-1 and tree node u at position prefix_len[b]+u
 *    (the depth-first KV-cache layout of "Tree Attention のカーネル融合",
 *    item 2, generalised to any parent-before-child numbering).
 *  - Target logits are [B][Tmax+1][V] fp32: row 0 belongs to the root, row
 *    1+u to node u.
 *  - Return value: TSD_OK or a negative TSD_ERR_* code for errors found on the
 *    host before any launch (nothing is launched then).  Errors found in the
 *    data on the device are OR-ed into *dev_status (TSD_DEV_* bits; pass NULL
 *    to ignore them); the caller reads that int32 when convenient.
 */
#ifndef TSD_H
#define TSD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st *tsd_stream_t;

#define TSD_MAX_TREE 128 /* largest Tmax (ancestor masks are 4 x u32) */

enum tsd_status {
    TSD_OK = 0,
    TSD_ERR_NULL = -1,        /* a required pointer is NULL                 */
    TSD_ERR_SHAPE = -2,       /* a size is out of range or inconsistent     */
    TSD_ERR_DTYPE = -3,       /* unsupported dtype / head_dim combination   */
    TSD_ERR_WORKSPACE = -4,   /* workspace smaller than *_workspace_size()  */
    TSD_ERR_CUDA = -5,        /* a CUDA runtime/driver call failed          */
    TSD_ERR_ALIGN = -6        /* a pointer is not 16-byte aligned           */
};

/* Bits OR-ed into *dev_status by the kernels. */
enum tsd_dev_status {
    TSD_DEV_BAD_TREE = 1,     /* n_nodes out of [0,Tmax] or parent[u] not in [-1,u-1] */
    TSD_DEV_BAD_TOKEN = 2,    /* a token id outside [0, V)                  */
    TSD_DEV_BAD_QROW = 4,     /* a q_row index outside [0, Rq)              */
    TSD_DEV_BAD_PREFIX = 8,   /* prefix_len[b] + n_nodes[b] > Lmax or < 0   */
    TSD_DEV_TIMEOUT = 16,     /* a bounded pipeline wait expired (kernel bailed out) */
    TSD_DEV_BAD_PATH = 32,    /* an accepted path that is not a valid commit list     */
    TSD_DEV_BAD_PAGE = 64,    /* a block-table entry outside [0, num_pages)          */
    TSD_DEV_BOUNDS = 128      /* checked build only (libtsd_checked.so): a kernel computed
                                 an index outside the buffer its arguments describe; the
                                 access was skipped                                    */
};

/* Element types of Q / K / V / attention output. */
enum tsd_dtype { TSD_F32 = 0, TSD_BF16 = 1 };

/* Attention kernels, as reported by tsd_tree_attention_plan. */
enum tsd_attention_path {
    TSD_PLAN_SIMT = 0,       /* CUDA cores, 16 query rows per CTA                       */
    TSD_PLAN_ROWS128 = 1,    /* tensor cores, 128-key tiles, one CTA per SM             */
    TSD_PLAN_ROWS64 = 2,     /* tensor cores, 64-key tiles, two CTAs per SM             */
    TSD_PLAN_KEYSPLIT = 3,   /* tensor cores, two softmax groups splitting the key tiles */
    TSD_PLAN_ROWS128_PAIRED = 4  /* 128-key tiles, two softmax warps per TMEM lane quarter */
};

/* Marker written to first_child[b][0] by tsd_tree_mask_build for a malformed
 * tree; the verify calls then report n_accepted[b] = -1 for that sequence. */
#define TSD_TREE_INVALID (-2)

/* Human-readable name of a tsd_status value. */
const char *tsd_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int tsd_version(void);

/* Number of kernels this library has launched in this process so far (all
 * devices, all streams).  Instrumentation for benchmarks. */
unsigned long long tsd_launch_count(void);

/*
 * Ancestor mask of each token tree (the topology-aware causal mask:
 * "トークンツリー構造の仕組み", last paragraph; "Tree Attention のカーネル融合",
 * item 1).
 *   parent       [B][Tmax] int32        node -> parent (-1 = root)
 *   n_nodes      [B] int32              T_b
 *   mask         [B][Tmax][W] uint32    out, W = ceil(Tmax/32): bit v of row u is
 *                                       set iff v is on the root->u path (u included)
 *   depth        [B][Tmax] int32        out, number of nodes on the root->u path
 *   first_child  [B][Tmax+1] int32      out, slot 0 = root, slot 1+c = node c:
 *                                       smallest child index or -1
 *   next_sibling [B][Tmax] int32        out, next larger index with the same parent, or -1
 * Every output slot is written: padding rows get mask 0, depth 0, links -1.
 * A malformed tree sets TSD_DEV_BAD_TREE, writes those padding values for the
 * whole sequence and first_child[b][0] = TSD_TREE_INVALID.
 * Host errors: TSD_ERR_NULL, TSD_ERR_SHAPE (B < 0, Tmax < 1 or > TSD_MAX_TREE).
 */
int tsd_tree_mask_build(const int32_t *parent, const int32_t *n_nodes, int B, int Tmax,
                        uint32_t *mask, int32_t *depth, int32_t *first_child,
                        int32_t *next_sibling, int32_t *dev_status, tsd_stream_t stream);

/*
 * Bytes of workspace tsd_tree_attention needs for these sizes (split-KV
 * partial results).  Depends only on the arguments and the current device.
 */
/*
 * The launch tsd_tree_attention would make for these sizes on a device with
 * num_sms SMs (host only, nothing is launched; the environment variables
 * that select the attention kernel are read as in the call itself):
 *   plan[0]  the kernel, a tsd_attention_path value
 *   plan[1]  query-row blocks per (sequence, KV head)
 *   plan[2]  key-range splits (combined by log-sum-exp when > 1)
 *   plan[3]  keys per split
 * Errors: TSD_ERR_NULL (plan), TSD_ERR_SHAPE (sizes as for the call,
 * num_sms < 1), TSD_ERR_DTYPE.
 */
int tsd_tree_attention_plan(int B, int Tmax, int Hq, int Hkv, int D, int Lmax, int dtype,
                            int num_sms, int32_t *plan);

size_t tsd_tree_attention_workspace_size(int B, int Tmax, int Hq, int Hkv, int D, int Lmax,
                                         int dtype);

/*
 * Tree attention ("トークンツリー構造の仕組み", equation
 * Attention(Q_u, K_{S_u}, V_{S_u})): for every node u < T_b and query head h,
 *   out[b][u][h] = sum_{j in S_u} softmax_j(scale * q[b][u][h] . k_j) v_j
 * where S_u = prefix positions 0..prefix_len[b]-1 plus the cache positions
 * prefix_len[b]+v of the nodes v whose bit is set in mask[b][u], and k_j, v_j
 * come from KV head h / (Hq / Hkv) (grouped-query attention).
 *   q            [B][Tmax][Hq][D]   dtype
 *   k_cache      [B][Hkv][Lmax][D]  dtype
 *   v_cache      [B][Hkv][Lmax][D]  dtype
 *   prefix_len   [B] int32          committed prefix length P_b
 *   n_nodes      [B] int32          T_b (prefix_len[b] + T_b <= Lmax)
 *   mask         [B][Tmax][W] uint32 from tsd_tree_mask_build
 *   out          [B][Tmax][Hq][D]   dtype; rows u >= T_b are not written
 * dtype TSD_BF16 (D = 64 or 128; fp32 accumulation and softmax) or TSD_F32.
 * Cache positions at or beyond prefix_len[b] + T_b are never read into the
 * result, whatever they hold.  q, k_cache, v_cache, out must be 16-byte
 * aligned.  Host errors: TSD_ERR_NULL, TSD_ERR_SHAPE (Hq % Hkv != 0, sizes
 * out of range, B * Hkv > 65535), TSD_ERR_DTYPE, TSD_ERR_ALIGN,
 * TSD_ERR_WORKSPACE, TSD_ERR_CUDA.
 * Device: TSD_DEV_BAD_PREFIX (that sequence's rows are not written),
 * TSD_DEV_TIMEOUT.
 * Kernel choice (results agree within the bf16 tolerance whichever runs):
 * bf16 with D = 128 and at least 8 packed query rows per KV head (Tmax *
 * Hq / Hkv) runs on the tensor cores -- 64-key tiles at two CTAs per SM up
 * to 128 packed rows, 128-key tiles at one CTA per SM above; everything else
 * on the CUDA cores.  The environment variables TSD_ATTN_ROWS_VARIANT=2
 * (64-key tiles above 128 rows too), TSD_ATTN_SMALL_VARIANT=keysplit (two
 * softmax groups splitting the key tiles, up to 128 rows) and
 * TSD_FORCE_PATH=simt (the CUDA-core kernel for every shape) select the
 * alternatives, and TSD_ATTN_SPLITS=n fixes the number of key-range splits
 * (at most 64 and one per key tile); they are read at every call.
 */
int tsd_tree_attention(const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *prefix_len, const int32_t *n_nodes, const uint32_t *mask,
                       int B, int Tmax, int Hq, int Hkv, int D, int Lmax, float scale,
                       int dtype, void *out, void *workspace, size_t workspace_bytes,
                       int32_t *dev_status, tsd_stream_t stream);

/*
 * Tree attention over a paged KV cache ("実運用への応用" / "vLLMとの関連" and the
 * outlook list: the tree verification combined with PagedAttention's
 * block-wise KV memory).  The same operation as tsd_tree_attention on the
 * logical cache the block table describes: logical position pos of sequence
 * b (prefix at 0..P_b-1, node u at P_b+u, as before) is row pos % page_size
 * of physical page block_table[b][pos / page_size].
 *   k_pages, v_pages  [num_pages][Hkv][page_size][D], dtype as for
 *                     tsd_tree_attention (caller-owned pools)
 *   block_table       [B][max_blocks] int32, physical page ids
 *   page_size         a power of two in [16, 4096]; the logical capacity is
 *                     max_blocks * page_size (the Lmax of the workspace size:
 *                     tsd_tree_attention_workspace_size(B, Tmax, Hq, Hkv, D,
 *                     max_blocks * page_size, dtype))
 * Entries of the table beyond a sequence's last key are never read.  An
 * entry outside [0, num_pages) for a key the sequence uses sets
 * TSD_DEV_BAD_PAGE (that key reads as zero, or as page 0 on the tensor-core
 * path).  Host errors: those of tsd_tree_attention, and TSD_ERR_SHAPE for a
 * page size that is not a power of two in range.
 */
int tsd_tree_attention_paged(const void *q, const void *k_pages, const void *v_pages,
                             const int32_t *block_table, int num_pages, int page_size,
                             int max_blocks, const int32_t *prefix_len, const int32_t *n_nodes,
                             const uint32_t *mask, int B, int Tmax, int Hq, int Hkv, int D,
                             float scale, int dtype, void *out, void *workspace,
                             size_t workspace_bytes, int32_t *dev_status, tsd_stream_t stream);

/* Bytes of workspace either verify call needs: a fixed ~40 KB (per-CTA
 * partial sums and barrier counters of the stochastic walk) plus 4 bytes per
 * logits row (greedy row argmax). */
size_t tsd_tree_verify_workspace_size(int B, int Tmax, int V);

/*
 * Greedy verification ("ツリー検証アルゴリズム", greedy variant): accept the
 * longest root path whose every token equals the argmax of its parent's
 * logits row (lowest token id on argmax ties; lowest terminal node index when
 * two paths are equally long), then append the argmax of the terminal's row
 * (row 0 when nothing is accepted).
 *   logits      [B][Tmax+1][V] fp32
 *   tokens      [B][Tmax] int32     speculated token of each node
 *   parent, n_nodes, mask, first_child   as produced / consumed above
 *   out_tokens  [B][Tmax+1] int32   out: accepted tokens, then the bonus token
 *   out_path    [B][Tmax] int32     out: accepted node indices, root-first
 *   n_accepted  [B] int32           out: number of accepted nodes (-1 if the
 *                                   sequence is malformed; nothing else written)
 * Entries beyond n_accepted (+1 for out_tokens) are not written.
 * Two forms give the same result: when the batch's logits (B (Tmax+1) V
 * floats) reach 64 MiB, one CTA per sequence walks the matched nodes level
 * by level and reads only the root row and the matched nodes' rows;
 * otherwise the argmax of every row with children is taken in parallel,
 * then the path.  TSD_GREEDY_FORM = "walk" or "rows" forces one (read at
 * every call).
 * Host errors: TSD_ERR_SHAPE (B < 0 or > 65535, Tmax, V < 1), TSD_ERR_NULL,
 * TSD_ERR_ALIGN (logits), TSD_ERR_WORKSPACE, TSD_ERR_CUDA.
 * Device: TSD_DEV_BAD_TOKEN.
 */
int tsd_tree_verify_greedy(const float *logits, const int32_t *tokens, const int32_t *parent,
                           const int32_t *n_nodes, const uint32_t *mask,
                           const int32_t *first_child, int B, int Tmax, int V,
                           int32_t *out_tokens, int32_t *out_path, int32_t *n_accepted,
                           void *workspace, size_t workspace_bytes, int32_t *dev_status,
                           tsd_stream_t stream);

/*
 * Stochastic verification by multi-step speculative sampling ("ツリー検証アル
 * ゴリズム": P_accept = min(1, P_LLM(x)/P_SSM(x)); on rejection
 * norm(max(0, P_LLM - P_SSM))).  Starting at the root, with p = softmax(l/T)
 * of the current node's row (fp64): the children are tried in ascending
 * index; child c with token x is accepted iff p(x) > 0 and
 * u_accept[b][c] * q(x) <= p(x), where q = q_probs[b][q_row[b][c]]; after a
 * rejection p becomes max(0, p - q) / sum(max(0, p - q)) (unchanged if that
 * sum is 0).  An accepted child becomes the current node.  When no child is
 * accepted (or there is none) the final token is drawn from p by inverse CDF:
 * the smallest token i whose ascending cumulative sum exceeds
 * u_sample[b][row], row being the current node's logits row (if rounding
 * leaves none: the largest i with p_i > 0).
 *   logits        [B][Tmax+1][V] fp32
 *   temperature   T > 0
 *   q_probs       [B][Rq][V] fp32   SSM distributions
 *   q_row         [B][Tmax] int32   row of q_probs that proposed node u
 *   tokens        [B][Tmax] int32
 *   n_nodes, first_child, next_sibling   from tsd_tree_mask_build
 *   u_accept      [B][Tmax] fp64, u_sample [B][Tmax+1] fp64: uniforms in (0,1)
 *   out_tokens, out_path, n_accepted      as for the greedy call
 * Work: one kernel launch; each sequence's walk reads only the logits rows
 * (and q rows) of the nodes it reaches.  The CTAs walking a sequence form a
 * thread-block cluster and exchange their partial sums through distributed
 * shared memory (V <= 32768), or are CTAs of a cooperative launch that
 * exchange them through the workspace; either way every wait is bounded
 * (about 2 s).  The environment variable TSD_WALK_EXCHANGE=global selects
 * the cooperative form for every V (read at every call).
 * Device: TSD_DEV_BAD_TOKEN, TSD_DEV_BAD_QROW, TSD_DEV_TIMEOUT (a barrier
 * wait expired; the affected sequences get n_accepted = -1).
 */
int tsd_tree_verify_stochastic(const float *logits, double temperature, const float *q_probs,
                               int Rq, const int32_t *q_row, const int32_t *tokens,
                               const int32_t *n_nodes, const int32_t *first_child,
                               const int32_t *next_sibling, const double *u_accept,
                               const double *u_sample, int B, int Tmax, int V,
                               int32_t *out_tokens, int32_t *out_path, int32_t *n_accepted,
                               void *workspace, size_t workspace_bytes, int32_t *dev_status,
                               tsd_stream_t stream);

/*
 * The grid tsd_tree_verify_stochastic (and its _noalloc form) launches for B
 * sequences over a vocabulary of V on the current device (host only,
 * nothing is launched; it reads the device's SM count and the walk kernel's
 * occupancy):
 *   plan[0]  teams: sequences walked at the same time (team t walks
 *            sequences t, t + teams, t + 2 teams, ...)
 *   plan[1]  CTAs per team, each owning one chunk of the vocabulary
 *   plan[2]  vocabulary entries per chunk
 *   plan[3]  CTAs in the launch (teams x CTAs per team)
 * A team is one thread-block cluster when V <= 32768 (then at most 8 CTAs)
 * and CTAs of a cooperative launch otherwise.
 * Errors: TSD_ERR_NULL (plan), TSD_ERR_SHAPE (B < 1, Tmax out of range,
 * V < 1), TSD_ERR_CUDA (no device or no cooperative launch).
 */
int tsd_tree_verify_stochastic_plan(int B, int Tmax, int V, int32_t *plan);

/* Forms of greedy verification, as reported by tsd_tree_verify_greedy_plan. */
enum tsd_greedy_form {
    TSD_GREEDY_WALK = 0,     /* one CTA per sequence walks the matched nodes            */
    TSD_GREEDY_ROWS = 1      /* the argmax of every row with children, then the path    */
};

/*
 * The form tsd_tree_verify_greedy takes for these sizes (host only, nothing
 * is launched; TSD_GREEDY_FORM is read as in the call itself): *form is a
 * tsd_greedy_form value.
 * Errors: TSD_ERR_NULL (form), TSD_ERR_SHAPE (B < 1, Tmax out of range, V < 1).
 */
int tsd_tree_verify_greedy_plan(int B, int Tmax, int V, int32_t *form);

/*
 * Token-tree construction ("マルチドラフトモデルアプローチ": item 1,
 * expansion-based trees <k_1, ..., k_n> take one SSM's top-k_i tokens at
 * every node of depth i-1; item 2, merge-based trees merge the outputs of
 * several SSMs into one token tree; "Tree Attention のカーネル融合", item 2: the
 * tree is laid out depth-first).  Tree arrays are those of the other calls:
 * parent, tokens, q_row [B][Tmax] int32, n_nodes [B] int32.
 *
 * tsd_tree_expand adds one level.  The frontier is the root when
 * n_nodes[b] == 0, else the nodes lvl_begin[b] .. n_nodes[b]-1 (the level
 * added last); frontier node i (in index order) has its SSM distribution in
 * q_probs[b][frow[b][i]] (q_probs [B][Rq][V] fp32, frow [B][Tmax] int32).
 * Each frontier node gets k children, appended in frontier order at
 * n_nodes + i*k + j, holding the k most probable tokens of its row in
 * descending probability (lower token id on ties), with q_row = frow[b][i];
 * then lvl_begin[b] = old n_nodes[b] and n_nodes[b] += F*k.  A level that
 * would exceed Tmax, a q row outside [0, Rq) or k > V changes nothing and
 * sets TSD_DEV_BAD_TREE.  Nodes come out level by level; renumber with
 * tsd_tree_dfs_order before the other calls if depth-first order is wanted.
 */
int tsd_tree_expand(const float *q_probs, int Rq, int V, const int32_t *frow, int k,
                    int32_t *parent, int32_t *tokens, int32_t *q_row, int32_t *n_nodes,
                    int32_t *lvl_begin, int B, int Tmax, int32_t *dev_status,
                    tsd_stream_t stream);

/*
 * tsd_tree_dfs_order renumbers each tree (any order in which parents precede
 * children) into depth-first pre-order, children in increasing old index:
 * perm[b][new] = old, out_parent / out_tokens / out_q_row renumbered
 * (entries beyond n_nodes untouched).  A malformed tree sets
 * TSD_DEV_BAD_TREE and writes nothing for that sequence.
 */
int tsd_tree_dfs_order(const int32_t *parent, const int32_t *tokens, const int32_t *q_row,
                       const int32_t *n_nodes, int B, int Tmax, int32_t *perm,
                       int32_t *out_parent, int32_t *out_tokens, int32_t *out_q_row,
                       int32_t *dev_status, tsd_stream_t stream);

/*
 * tsd_tree_merge_chains builds the tree from M chains per sequence: chain m
 * proposes chain_tokens[b][m][0 .. chain_len[b][m]-1], step i drawn from q row
 * chain_q_row[b][m][i] ([B][M][L] int32, lengths [B][M]).  A chain reuses
 * earlier nodes while its prefix matches (same parent, same token) and
 * creates nodes from its first difference on; a node keeps the q row of the
 * chain that created it.  Output in depth-first pre-order, children in
 * creation order; n_nodes[b] = the node count, or -1 (with
 * TSD_DEV_BAD_TREE) when the tree would exceed Tmax or a length is outside
 * [0, L].
 */
int tsd_tree_merge_chains(const int32_t *chain_tokens, const int32_t *chain_q_row,
                          const int32_t *chain_len, int M, int L, int B, int Tmax,
                          int32_t *parent, int32_t *tokens, int32_t *q_row, int32_t *n_nodes,
                          int32_t *dev_status, tsd_stream_t stream);

/*
 * Commit of the accepted path ("Tree Attention のカーネル融合", item 2: the
 * tree's KV entries stay consistent with the existing KV cache; the
 * flatkey.ai guide's verification diagram: the accepted prefix is committed).
 * For every sequence b with n = n_accepted[b] >= 0 and accepted nodes
 * u_i = out_path[b][i] (i < n, as the verify calls write them), the K and V
 * rows of every KV head at cache position P_b + u_i move to P_b + i, in place,
 * all at once (no row is written before every source has been read), and
 * new_prefix_len[b] = P_b + n.  The final sampled token has no KV entry yet.
 *   k_cache, v_cache  [B][Hkv][Lmax][D] (dtype TSD_BF16 or TSD_F32), in/out
 *   prefix_len        [B] int32, P_b before the commit
 *   out_path          [B][Tmax] int32, n_accepted [B] int32 (verify outputs)
 *   new_prefix_len    [B] int32, out (P_b for a skipped sequence)
 * Sequences with n_accepted < 0 are skipped silently (their verify call
 * already reported why).  A path that is not strictly increasing, leaves
 * [0, Tmax), is longer than Tmax or reaches past Lmax moves nothing and sets
 * TSD_DEV_BAD_PATH.  Pointers 16-byte aligned; D * element size a multiple
 * of 16 and at most 512 bytes; B at most 65535.  Host errors: TSD_ERR_NULL,
 * TSD_ERR_SHAPE, TSD_ERR_DTYPE, TSD_ERR_ALIGN, TSD_ERR_CUDA.  Device:
 * TSD_DEV_BAD_PATH.
 */
int tsd_kv_commit(void *k_cache, void *v_cache, const int32_t *prefix_len,
                  const int32_t *out_path, const int32_t *n_accepted, int B, int Tmax, int Hkv,
                  int D, int Lmax, int dtype, int32_t *new_prefix_len, int32_t *dev_status,
                  tsd_stream_t stream);

/*
 * Self-test of the bounded waits (no counterpart in the paper).  Every wait
 * in the kernels above gives up after a time limit, sets TSD_DEV_TIMEOUT and
 * returns, so that a stalled pipeline ends with a status instead of a hung
 * GPU.  This call runs those same wait routines on something that never
 * completes, with a short limit, so that tests can check the behaviour:
 *   kind 0  the mbarrier wait of the tensor-core attention kernels, on an
 *           mbarrier nobody arrives on;
 *   kind 1  the team barrier of the stochastic walk, on a counter whose
 *           target one CTA cannot reach;
 *   kind 2  the cluster exchange of the stochastic walk (thread-block
 *           cluster teams), in a cluster of two CTAs of which one never
 *           takes part.
 *   limit_ns  in [1 ms, 2 s]; scratch: 8 bytes of device memory (8-aligned;
 *           unused by kind 2).
 * Expected result: the kernel ends after about limit_ns with TSD_DEV_TIMEOUT
 * set in *dev_status.  Host errors: TSD_ERR_SHAPE, TSD_ERR_NULL,
 * TSD_ERR_ALIGN, TSD_ERR_CUDA.
 */
int tsd_debug_wait_probe(int kind, unsigned long long limit_ns, void *scratch,
                         int32_t *dev_status, tsd_stream_t stream);

/*
 * Stochastic verification without a workspace, for callers that cannot
 * allocate device memory (for example a serving engine whose KV-cache pool
 * already owns nearly all of the GPU's memory, or a caller reaching the
 * library through a plain C interface with no device allocator).  The paper
 * has no counterpart to this call; it is the same operation as
 * tsd_tree_verify_stochastic, with the same arguments minus the workspace.
 *
 * The scratch it needs lives in a fixed array of TSD_NOALLOC_SCRATCH_BYTES
 * inside the library's device code; every GPU that loads the library holds
 * that array until the process exits.  Nothing is allocated: no cudaMalloc,
 * no cudaFree, no allocating library routine.
 *   - The scratch it needs is fixed (about 40 KB: the per-CTA partial sums
 *     and barrier counters of the walk), whatever B, Tmax and V are, so no
 *     shape is refused for size; TSD_ERR_WORKSPACE would mean a build whose
 *     array is smaller than that, and then nothing is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents.  Calls whose kernels may overlap on the GPU (different
 *     streams, or concurrent host threads) race on it: serialise them.
 */
#define TSD_NOALLOC_SCRATCH_BYTES (1u << 16)

int tsd_tree_verify_stochastic_noalloc(const float *logits, double temperature,
                                       const float *q_probs, int Rq, const int32_t *q_row,
                                       const int32_t *tokens, const int32_t *n_nodes,
                                       const int32_t *first_child, const int32_t *next_sibling,
                                       const double *u_accept, const double *u_sample, int B,
                                       int Tmax, int V, int32_t *out_tokens, int32_t *out_path,
                                       int32_t *n_accepted, int32_t *dev_status,
                                       tsd_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TSD_H */
