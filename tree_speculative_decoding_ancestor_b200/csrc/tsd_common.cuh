// Device helpers shared by the libtsd kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include "tsd.h"

namespace tsd {

constexpr int kMaxTree = TSD_MAX_TREE;
constexpr int kMaskWords = (TSD_MAX_TREE + 31) / 32;

__device__ __forceinline__ void flag(int32_t *dev_status, int bits)
{
    if (dev_status)
        atomicOr(dev_status, bits);
}

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_float(float x);
template <> __device__ __forceinline__ float from_float<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float x)
{
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Bounds checks of the checked build.  Compiled with -DTSD_CHECKS (the
// library libtsd_checked.so, for small-case debugging), every global access
// whose index a kernel computes is first compared with the extent of the
// buffer the call's arguments describe; an index outside it sets
// TSD_DEV_BOUNDS in the status word and the access is skipped (nothing
// traps).  In the normal build in_bounds() is constant true and the checks
// compile away.
#ifdef TSD_CHECKS
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

__device__ __forceinline__ bool in_bounds(long long i, long long n, int32_t *dev_status)
{
    if (!kChecked)
        return true;
    if (i >= 0 && i < n)
        return true;
    flag(dev_status, TSD_DEV_BOUNDS);
    return false;
}

// Sequence-level validity shared by the attention and verify kernels.
__device__ __forceinline__ bool tree_header_ok(int T, int Tmax) { return T >= 0 && T <= Tmax; }

}  // namespace tsd

// Host-side launch helpers.

// Every C-ABI call that launches work shows up as a range named after the
// entry point on a profiler's timeline (NVTX; without an attached tool the
// push and pop cost a call each and record nothing).
namespace tsd {
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
}  // namespace tsd
#define TSD_NVTX_RANGE() tsd::NvtxRange tsd_nvtx_range_(__func__)

#define TSD_CUDA_TRY(expr)                                                                    \
    do {                                                                                      \
        cudaError_t e_ = (expr);                                                              \
        if (e_ != cudaSuccess)                                                                \
            return TSD_ERR_CUDA;                                                              \
    } while (0)

// Checks the launch just made and counts it.
#define TSD_LAUNCH_CHECK()                                                                    \
    do {                                                                                      \
        if (cudaPeekAtLastError() != cudaSuccess) {                                           \
            (void)cudaGetLastError();                                                         \
            return TSD_ERR_CUDA;                                                              \
        }                                                                                     \
        tsd::count_launch();                                                                  \
    } while (0)

// Internal launchers (defined in the kernel files, called by capi.cu).
namespace tsd {
void count_launch();
int launch_tree_mask(const int32_t *parent, const int32_t *n_nodes, int B, int Tmax,
                     uint32_t *mask, int32_t *depth, int32_t *first_child, int32_t *next_sibling,
                     int32_t *dev_status, cudaStream_t stream);

// Where K/V row `pos` of (sequence b, KV head hk) lives.  table == nullptr:
// a contiguous cache [B][Hkv][Lmax][D].  Otherwise a paged pool
// [num_pages][Hkv][page_size][D]: logical page pos / page_size of sequence b
// is physical page table[b][pos / page_size] (page_size a power of two).
struct KvPages {
    const int32_t *table = nullptr;
    int max_blocks = 0, page_size = 0, log2_page = 0, num_pages = 0;
};

// Row index (in rows of D elements) of K/V position `pos`; a page id outside
// [0, num_pages) yields -1.
__device__ __forceinline__ long long kv_row(const KvPages &pg, int b, int hk, int Hkv, int Lmax,
                                            int pos)
{
    if (!pg.table)
        return ((long long)b * Hkv + hk) * Lmax + pos;
    const int page = pg.table[(size_t)b * pg.max_blocks + (pos >> pg.log2_page)];
    if (page < 0 || page >= pg.num_pages)
        return -1;
    return ((long long)page * Hkv + hk) * pg.page_size + (pos & (pg.page_size - 1));
}

// Rows of D elements the K (or V) buffer holds: the contiguous cache
// [B][Hkv][Lmax] or the paged pool [num_pages][Hkv][page_size] (for the
// checked build's bounds).
__host__ __device__ __forceinline__ long long kv_rows_total(const KvPages &pg, int B, int Hkv,
                                                            int Lmax)
{
    return pg.table ? (long long)pg.num_pages * Hkv * pg.page_size : (long long)B * Hkv * Lmax;
}

struct AttnArgs {
    const void *q, *k, *v;
    const int32_t *prefix_len, *n_nodes;
    const uint32_t *mask;
    int B, Tmax, Hq, Hkv, D, Lmax, dtype;   // Lmax: logical capacity (max_blocks * page_size if paged)
    float scale;
    void *out;
    int32_t *dev_status;
    KvPages pages;
};
size_t simt_attention_workspace(const AttnArgs &a, int num_sms);
void simt_attention_plan(const AttnArgs &a, int num_sms, int32_t out[4]);
void umma_attention_plan(const AttnArgs &a, int num_sms, int32_t out[4]);
int launch_simt_attention(const AttnArgs &a, void *ws, size_t ws_bytes, int num_sms,
                          cudaStream_t stream);
bool umma_attention_supported(const AttnArgs &a);
size_t umma_attention_workspace(const AttnArgs &a, int num_sms);
int launch_umma_attention(const AttnArgs &a, void *ws, size_t ws_bytes, int num_sms,
                          cudaStream_t stream);

size_t verify_workspace(int B, int Tmax, int V);
size_t verify_stochastic_scratch();   // fixed: independent of the shape
int verify_stochastic_plan(int B, int V, int32_t out[4]);   // teams, K, chunk, CTAs
int launch_tree_expand(const float *q_probs, int Rq, int V, const int32_t *frow, int k,
                       int32_t *parent, int32_t *tokens, int32_t *q_row, int32_t *n_nodes,
                       int32_t *lvl_begin, int B, int Tmax, int32_t *dev_status,
                       cudaStream_t stream);
int launch_tree_dfs(const int32_t *parent, const int32_t *tokens, const int32_t *q_row,
                    const int32_t *n_nodes, int B, int Tmax, int32_t *perm, int32_t *out_parent,
                    int32_t *out_tokens, int32_t *out_q_row, int32_t *dev_status,
                    cudaStream_t stream);
int launch_tree_merge(const int32_t *ctok, const int32_t *cq, const int32_t *clen, int M, int L,
                      int B, int Tmax, int32_t *parent, int32_t *tokens, int32_t *q_row,
                      int32_t *n_nodes, int32_t *dev_status, cudaStream_t stream);
int launch_wait_probe(int kind, unsigned long long limit_ns, void *scratch,
                      int32_t *dev_status, cudaStream_t stream);
int launch_kv_commit(void *k_cache, void *v_cache, const int32_t *prefix_len,
                     const int32_t *out_path, const int32_t *n_accepted, int B, int Tmax, int Hkv,
                     int Lmax, int row_bytes, int32_t *new_prefix, int32_t *dev_status,
                     cudaStream_t stream);
// true: greedy verification takes the all-rows scan for these sizes (else
// the walk over matched nodes); reads TSD_GREEDY_FORM.
bool greedy_all_rows(int B, int Tmax, int V);

int launch_verify_greedy(const float *logits, const int32_t *tokens, const int32_t *parent,
                         const int32_t *n_nodes, const uint32_t *mask,
                         const int32_t *first_child, int B, int Tmax, int V,
                         int32_t *out_tokens, int32_t *out_path, int32_t *n_accepted, void *ws,
                         int32_t *dev_status, cudaStream_t stream);
int launch_verify_stochastic(const float *logits, double temperature, const float *q_probs,
                             int Rq, const int32_t *q_row, const int32_t *tokens,
                             const int32_t *n_nodes, const int32_t *first_child,
                             const int32_t *next_sibling, const double *u_accept,
                             const double *u_sample, int B, int Tmax, int V,
                             int32_t *out_tokens, int32_t *out_path, int32_t *n_accepted,
                             void *ws, int32_t *dev_status, cudaStream_t stream);
}  // namespace tsd
