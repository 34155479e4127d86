// extern "C" entry points of libtsd: argument checks on the host, then the
// launches.  Nothing here allocates device memory or synchronizes.
#include <atomic>
#include <cstdint>
#include <cstdlib>

#include "tsd_common.cuh"

namespace tsd {
static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace tsd

namespace {

int device_sms()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return sms;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;
    return sms;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Largest y extent of a launch grid: the attention kernels run (b, KV head)
// pairs on y, the greedy row kernel and the commit kernel the sequences.
constexpr long long kMaxGridY = 65535;

// Path selection for tree attention: the tensor-core kernel when the packed
// query block is large enough and the layout fits it, otherwise CUDA cores.
// TSD_FORCE_PATH=simt|umma overrides (for A/B measurement).
int choose_umma(const tsd::AttnArgs &a)
{
    const char *force = std::getenv("TSD_FORCE_PATH");
    const bool ok = tsd::umma_attention_supported(a);
    if (force && force[0] == 's')
        return 0;
    if (force && force[0] == 'u')
        return ok ? 1 : 0;
    return ok ? 1 : 0;
}

int check_attn(const tsd::AttnArgs &a)
{
    if (!a.q || !a.k || !a.v || !a.prefix_len || !a.n_nodes || !a.mask || !a.out)
        return TSD_ERR_NULL;
    if (a.B < 0 || a.Tmax < 1 || a.Tmax > TSD_MAX_TREE || a.Hq < 1 || a.Hkv < 1 ||
        a.Hq % a.Hkv != 0 || a.Lmax < a.Tmax || (long long)a.B * a.Hkv > kMaxGridY)
        return TSD_ERR_SHAPE;
    if (a.dtype != TSD_F32 && a.dtype != TSD_BF16)
        return TSD_ERR_DTYPE;
    if (a.D != 64 && a.D != 128)
        return TSD_ERR_DTYPE;
    if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.out))
        return TSD_ERR_ALIGN;
    return TSD_OK;
}

}  // namespace

extern "C" {

const char *tsd_status_string(int status)
{
    switch (status) {
    case TSD_OK: return "ok";
    case TSD_ERR_NULL: return "a required pointer is NULL";
    case TSD_ERR_SHAPE: return "size out of range or inconsistent";
    case TSD_ERR_DTYPE: return "unsupported dtype / head_dim";
    case TSD_ERR_WORKSPACE: return "workspace too small";
    case TSD_ERR_CUDA: return "CUDA call failed";
    case TSD_ERR_ALIGN: return "pointer not 16-byte aligned";
    default: return "unknown status";
    }
}

int tsd_version(void) { return 101; }

unsigned long long tsd_launch_count(void) { return tsd::g_launches.load(); }

int tsd_tree_mask_build(const int32_t *parent, const int32_t *n_nodes, int B, int Tmax,
                        uint32_t *mask, int32_t *depth, int32_t *first_child,
                        int32_t *next_sibling, int32_t *dev_status, tsd_stream_t stream)
{
    TSD_NVTX_RANGE();
    if (B < 0 || Tmax < 1 || Tmax > TSD_MAX_TREE)
        return TSD_ERR_SHAPE;
    if (B == 0)
        return TSD_OK;
    if (!parent || !n_nodes || !mask || !depth || !first_child || !next_sibling)
        return TSD_ERR_NULL;
    return tsd::launch_tree_mask(parent, n_nodes, B, Tmax, mask, depth, first_child, next_sibling,
                                 dev_status, reinterpret_cast<cudaStream_t>(stream));
}

size_t tsd_tree_attention_workspace_size(int B, int Tmax, int Hq, int Hkv, int D, int Lmax,
                                         int dtype)
{
    tsd::AttnArgs a{};
    a.B = B; a.Tmax = Tmax; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.Lmax = Lmax; a.dtype = dtype;
    if (B <= 0 || Tmax < 1 || Tmax > TSD_MAX_TREE || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 ||
        (D != 64 && D != 128) || Lmax < Tmax || (long long)B * Hkv > kMaxGridY)
        return 0;
    const int sms = device_sms();
    return choose_umma(a) ? tsd::umma_attention_workspace(a, sms)
                          : tsd::simt_attention_workspace(a, sms);
}

int tsd_tree_attention_plan(int B, int Tmax, int Hq, int Hkv, int D, int Lmax, int dtype,
                            int num_sms, int32_t *plan)
{
    if (!plan)
        return TSD_ERR_NULL;
    if (B < 1 || Tmax < 1 || Tmax > TSD_MAX_TREE || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 ||
        Lmax < Tmax || num_sms < 1 || (long long)B * Hkv > kMaxGridY)
        return TSD_ERR_SHAPE;
    if ((dtype != TSD_F32 && dtype != TSD_BF16) || (D != 64 && D != 128))
        return TSD_ERR_DTYPE;
    tsd::AttnArgs a{};
    a.B = B; a.Tmax = Tmax; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.Lmax = Lmax; a.dtype = dtype;
    if (choose_umma(a))
        tsd::umma_attention_plan(a, num_sms, plan);
    else
        tsd::simt_attention_plan(a, num_sms, plan);
    return TSD_OK;
}

int tsd_tree_attention(const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *prefix_len, const int32_t *n_nodes, const uint32_t *mask,
                       int B, int Tmax, int Hq, int Hkv, int D, int Lmax, float scale,
                       int dtype, void *out, void *workspace, size_t workspace_bytes,
                       int32_t *dev_status, tsd_stream_t stream)
{
    TSD_NVTX_RANGE();
    tsd::AttnArgs a;
    a.q = q; a.k = k_cache; a.v = v_cache; a.prefix_len = prefix_len; a.n_nodes = n_nodes;
    a.mask = mask; a.B = B; a.Tmax = Tmax; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.Lmax = Lmax;
    a.dtype = dtype; a.scale = scale; a.out = out; a.dev_status = dev_status;
    if (B == 0)
        return TSD_OK;
    const int rc = check_attn(a);
    if (rc != TSD_OK)
        return rc;
    const int sms = device_sms();
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (choose_umma(a)) {
        if (workspace_bytes < tsd::umma_attention_workspace(a, sms))
            return TSD_ERR_WORKSPACE;
        return tsd::launch_umma_attention(a, workspace, workspace_bytes, sms, s);
    }
    if (workspace_bytes < tsd::simt_attention_workspace(a, sms))
        return TSD_ERR_WORKSPACE;
    return tsd::launch_simt_attention(a, workspace, workspace_bytes, sms, s);
}

int tsd_tree_attention_paged(const void *q, const void *k_pages, const void *v_pages,
                             const int32_t *block_table, int num_pages, int page_size,
                             int max_blocks, const int32_t *prefix_len, const int32_t *n_nodes,
                             const uint32_t *mask, int B, int Tmax, int Hq, int Hkv, int D,
                             float scale, int dtype, void *out, void *workspace,
                             size_t workspace_bytes, int32_t *dev_status, tsd_stream_t stream)
{
    TSD_NVTX_RANGE();
    if (page_size < 16 || page_size > 4096 || (page_size & (page_size - 1)) != 0 ||
        max_blocks < 1 || num_pages < 1 || (long long)max_blocks * page_size > (1LL << 30))
        return TSD_ERR_SHAPE;
    tsd::AttnArgs a;
    a.q = q; a.k = k_pages; a.v = v_pages; a.prefix_len = prefix_len; a.n_nodes = n_nodes;
    a.mask = mask; a.B = B; a.Tmax = Tmax; a.Hq = Hq; a.Hkv = Hkv; a.D = D;
    a.Lmax = max_blocks * page_size;
    a.dtype = dtype; a.scale = scale; a.out = out; a.dev_status = dev_status;
    a.pages.table = block_table;
    a.pages.max_blocks = max_blocks;
    a.pages.page_size = page_size;
    a.pages.log2_page = __builtin_ctz((unsigned)page_size);
    a.pages.num_pages = num_pages;
    if (B == 0)
        return TSD_OK;
    if (!block_table)
        return TSD_ERR_NULL;
    const int rc = check_attn(a);
    if (rc != TSD_OK)
        return rc;
    const int sms = device_sms();
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (choose_umma(a)) {
        if (workspace_bytes < tsd::umma_attention_workspace(a, sms))
            return TSD_ERR_WORKSPACE;
        return tsd::launch_umma_attention(a, workspace, workspace_bytes, sms, s);
    }
    if (workspace_bytes < tsd::simt_attention_workspace(a, sms))
        return TSD_ERR_WORKSPACE;
    return tsd::launch_simt_attention(a, workspace, workspace_bytes, sms, s);
}

size_t tsd_tree_verify_workspace_size(int B, int Tmax, int V)
{
    if (B <= 0 || Tmax < 1 || Tmax > TSD_MAX_TREE || V < 1)
        return 0;
    return tsd::verify_workspace(B, Tmax, V);
}

int tsd_tree_verify_greedy(const float *logits, const int32_t *tokens, const int32_t *parent,
                           const int32_t *n_nodes, const uint32_t *mask,
                           const int32_t *first_child, int B, int Tmax, int V,
                           int32_t *out_tokens, int32_t *out_path, int32_t *n_accepted,
                           void *workspace, size_t workspace_bytes, int32_t *dev_status,
                           tsd_stream_t stream)
{
    TSD_NVTX_RANGE();
    if (B < 0 || B > kMaxGridY || Tmax < 1 || Tmax > TSD_MAX_TREE || V < 1)
        return TSD_ERR_SHAPE;
    if (B == 0)
        return TSD_OK;
    if (!logits || !tokens || !parent || !n_nodes || !mask || !first_child || !out_tokens ||
        !out_path || !n_accepted || !workspace)
        return TSD_ERR_NULL;
    if (!aligned16(logits))
        return TSD_ERR_ALIGN;
    if (workspace_bytes < tsd::verify_workspace(B, Tmax, V))
        return TSD_ERR_WORKSPACE;
    return tsd::launch_verify_greedy(logits, tokens, parent, n_nodes, mask, first_child, B, Tmax,
                                     V, out_tokens, out_path, n_accepted, workspace, dev_status,
                                     reinterpret_cast<cudaStream_t>(stream));
}

int tsd_tree_verify_stochastic(const float *logits, double temperature, const float *q_probs,
                               int Rq, const int32_t *q_row, const int32_t *tokens,
                               const int32_t *n_nodes, const int32_t *first_child,
                               const int32_t *next_sibling, const double *u_accept,
                               const double *u_sample, int B, int Tmax, int V,
                               int32_t *out_tokens, int32_t *out_path, int32_t *n_accepted,
                               void *workspace, size_t workspace_bytes, int32_t *dev_status,
                               tsd_stream_t stream)
{
    TSD_NVTX_RANGE();
    if (B < 0 || Tmax < 1 || Tmax > TSD_MAX_TREE || V < 1 || Rq < 1 || !(temperature > 0.0))
        return TSD_ERR_SHAPE;
    if (B == 0)
        return TSD_OK;
    if (!logits || !q_probs || !q_row || !tokens || !n_nodes || !first_child || !next_sibling ||
        !u_accept || !u_sample || !out_tokens || !out_path || !n_accepted || !workspace)
        return TSD_ERR_NULL;
    if (!aligned16(logits) || !aligned16(q_probs))
        return TSD_ERR_ALIGN;
    if (workspace_bytes < tsd::verify_workspace(B, Tmax, V))
        return TSD_ERR_WORKSPACE;
    return tsd::launch_verify_stochastic(logits, temperature, q_probs, Rq, q_row, tokens, n_nodes,
                                         first_child, next_sibling, u_accept, u_sample, B, Tmax,
                                         V, out_tokens, out_path, n_accepted, workspace,
                                         dev_status, reinterpret_cast<cudaStream_t>(stream));
}

int tsd_tree_verify_stochastic_plan(int B, int Tmax, int V, int32_t *plan)
{
    if (!plan)
        return TSD_ERR_NULL;
    if (B < 1 || Tmax < 1 || Tmax > TSD_MAX_TREE || V < 1)
        return TSD_ERR_SHAPE;
    return tsd::verify_stochastic_plan(B, V, plan);
}

int tsd_tree_verify_greedy_plan(int B, int Tmax, int V, int32_t *form)
{
    if (!form)
        return TSD_ERR_NULL;
    if (B < 1 || Tmax < 1 || Tmax > TSD_MAX_TREE || V < 1)
        return TSD_ERR_SHAPE;
    *form = tsd::greedy_all_rows(B, Tmax, V) ? TSD_GREEDY_ROWS : TSD_GREEDY_WALK;
    return TSD_OK;
}

int tsd_kv_commit(void *k_cache, void *v_cache, const int32_t *prefix_len,
                  const int32_t *out_path, const int32_t *n_accepted, int B, int Tmax, int Hkv,
                  int D, int Lmax, int dtype, int32_t *new_prefix_len, int32_t *dev_status,
                  tsd_stream_t stream)
{
    TSD_NVTX_RANGE();
    if (B < 0 || B > kMaxGridY || Tmax < 1 || Tmax > TSD_MAX_TREE || Hkv < 1 || D < 1 ||
        Lmax < 1)
        return TSD_ERR_SHAPE;
    if (dtype != TSD_F32 && dtype != TSD_BF16)
        return TSD_ERR_DTYPE;
    const int row_bytes = D * (dtype == TSD_F32 ? 4 : 2);
    if (row_bytes % 16 != 0 || row_bytes > 512)
        return TSD_ERR_SHAPE;
    if (B == 0)
        return TSD_OK;
    if (!k_cache || !v_cache || !prefix_len || !out_path || !n_accepted || !new_prefix_len)
        return TSD_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(k_cache) & 15u) || (reinterpret_cast<uintptr_t>(v_cache) & 15u))
        return TSD_ERR_ALIGN;
    return tsd::launch_kv_commit(k_cache, v_cache, prefix_len, out_path, n_accepted, B, Tmax,
                                 Hkv, Lmax, row_bytes, new_prefix_len, dev_status,
                                 reinterpret_cast<cudaStream_t>(stream));
}

int tsd_tree_expand(const float *q_probs, int Rq, int V, const int32_t *frow, int k,
                    int32_t *parent, int32_t *tokens, int32_t *q_row, int32_t *n_nodes,
                    int32_t *lvl_begin, int B, int Tmax, int32_t *dev_status,
                    tsd_stream_t stream)
{
    TSD_NVTX_RANGE();
    if (B < 0 || Tmax < 1 || Tmax > TSD_MAX_TREE || Rq < 1 || V < 1 || k < 1 || k > Tmax)
        return TSD_ERR_SHAPE;
    if (B == 0)
        return TSD_OK;
    if (!q_probs || !frow || !parent || !tokens || !q_row || !n_nodes || !lvl_begin)
        return TSD_ERR_NULL;
    return tsd::launch_tree_expand(q_probs, Rq, V, frow, k, parent, tokens, q_row, n_nodes,
                                   lvl_begin, B, Tmax, dev_status,
                                   reinterpret_cast<cudaStream_t>(stream));
}

int tsd_tree_dfs_order(const int32_t *parent, const int32_t *tokens, const int32_t *q_row,
                       const int32_t *n_nodes, int B, int Tmax, int32_t *perm,
                       int32_t *out_parent, int32_t *out_tokens, int32_t *out_q_row,
                       int32_t *dev_status, tsd_stream_t stream)
{
    TSD_NVTX_RANGE();
    if (B < 0 || Tmax < 1 || Tmax > TSD_MAX_TREE)
        return TSD_ERR_SHAPE;
    if (B == 0)
        return TSD_OK;
    if (!parent || !tokens || !q_row || !n_nodes || !perm || !out_parent || !out_tokens ||
        !out_q_row)
        return TSD_ERR_NULL;
    return tsd::launch_tree_dfs(parent, tokens, q_row, n_nodes, B, Tmax, perm, out_parent,
                                out_tokens, out_q_row, dev_status,
                                reinterpret_cast<cudaStream_t>(stream));
}

int tsd_tree_merge_chains(const int32_t *chain_tokens, const int32_t *chain_q_row,
                          const int32_t *chain_len, int M, int L, int B, int Tmax,
                          int32_t *parent, int32_t *tokens, int32_t *q_row, int32_t *n_nodes,
                          int32_t *dev_status, tsd_stream_t stream)
{
    TSD_NVTX_RANGE();
    if (B < 0 || M < 1 || L < 1 || Tmax < 1 || Tmax > TSD_MAX_TREE)
        return TSD_ERR_SHAPE;
    if (B == 0)
        return TSD_OK;
    if (!chain_tokens || !chain_q_row || !chain_len || !parent || !tokens || !q_row || !n_nodes)
        return TSD_ERR_NULL;
    return tsd::launch_tree_merge(chain_tokens, chain_q_row, chain_len, M, L, B, Tmax, parent,
                                  tokens, q_row, n_nodes, dev_status,
                                  reinterpret_cast<cudaStream_t>(stream));
}

int tsd_debug_wait_probe(int kind, unsigned long long limit_ns, void *scratch,
                         int32_t *dev_status, tsd_stream_t stream)
{
    TSD_NVTX_RANGE();
    if (kind < 0 || kind > 2 || limit_ns < 1000000ull || limit_ns > 2000000000ull)
        return TSD_ERR_SHAPE;
    if (!scratch || !dev_status)
        return TSD_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(scratch) & 7u)
        return TSD_ERR_ALIGN;
    return tsd::launch_wait_probe(kind, limit_ns, scratch, dev_status,
                                  reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
