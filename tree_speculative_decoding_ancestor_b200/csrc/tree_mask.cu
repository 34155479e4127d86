// Ancestor-mask builder: the topology-aware causal mask of SpecInfer's tree
// attention ("トークンツリー構造の仕組み": node u attends only to the nodes on
// its root path S_u; "Tree Attention のカーネル融合", item 1: the mask is
// precomputed from the tree topology).
//
// One CTA of 128 threads per sequence, one thread per node slot.  The parent
// array (<= 512 B) is staged in shared memory (read beside the node count,
// one global round trip); every node walks its own root path there (<= 128
// steps, bounded because parent[v] < v is validated first).  Child lists
// come from one 128-bit set of children per node: the first child is its
// lowest bit, a node's next sibling the next bit set above its own.
#include <climits>

#include "tsd_common.cuh"

namespace tsd {

__global__ void __launch_bounds__(kMaxTree)
    tree_mask_kernel(const int32_t *__restrict__ parent, const int32_t *__restrict__ n_nodes,
                     int Tmax, int W, uint32_t *__restrict__ mask, int32_t *__restrict__ depth,
                     int32_t *__restrict__ first_child, int32_t *__restrict__ next_sibling,
                     int32_t *dev_status)
{
    __shared__ int32_t par[kMaxTree];
    __shared__ uint32_t kids[kMaxTree + 1][kMaskWords];   // children of node v - 1 (v = 0: root)
    const int b = blockIdx.x;
    const int u = threadIdx.x;
    const long long nb = (long long)gridDim.x * Tmax;   // B * Tmax
    // both reads at once: the slots past the node count are dropped below
    int p = -1;
    if (u < Tmax && in_bounds((long long)b * Tmax + u, nb, dev_status))
        p = parent[(size_t)b * Tmax + u];
    const int T = n_nodes[b];
    const bool bad_T = !tree_header_ok(T, Tmax);
    if (bad_T || u >= T)
        p = -1;
    par[u] = p;
    for (int s = u; s <= kMaxTree; s += blockDim.x)
#pragma unroll
        for (int w = 0; w < kMaskWords; ++w)
            kids[s][w] = 0u;
    const bool bad_u = !bad_T && u < T && (p < -1 || p >= u);
    const bool bad = __syncthreads_or(bad_T || bad_u);

    uint32_t m[kMaskWords] = {0u, 0u, 0u, 0u};
    int d = 0;
    if (!bad && u < T) {
        for (int v = u; v >= 0; v = par[v]) {
            m[v >> 5] |= 1u << (v & 31);
            ++d;
        }
        atomicOr(&kids[p + 1][u >> 5], 1u << (u & 31));
    }
    __syncthreads();
    // the lowest child above index `after` in set s (-1: none)
    auto next_kid = [&](int s, int after) {
        for (int w = (after + 1) >> 5; w < kMaskWords; ++w) {
            uint32_t bits = kids[s][w];
            if (w == (after + 1) >> 5)
                bits &= ~0u << ((after + 1) & 31);
            if (bits)
                return w * 32 + __ffs(bits) - 1;
        }
        return -1;
    };
    int ns = -1;
    if (!bad && u < T && u + 1 < kMaxTree)
        ns = next_kid(p + 1, u);
    if (u < Tmax && in_bounds((long long)b * Tmax + u, nb, dev_status)) {
        for (int w = 0; w < W; ++w)
            if (in_bounds(((long long)b * Tmax + u) * W + w, nb * W, dev_status))
                mask[((size_t)b * Tmax + u) * W + w] = m[w];
        depth[(size_t)b * Tmax + u] = d;
        next_sibling[(size_t)b * Tmax + u] = ns;
    }
    for (int s = u; s <= Tmax; s += blockDim.x) {
        int v = bad ? -1 : next_kid(s, -1);
        if (bad && s == 0)
            v = TSD_TREE_INVALID;
        if (in_bounds((long long)b * (Tmax + 1) + s, (long long)gridDim.x * (Tmax + 1),
                      dev_status))
            first_child[(size_t)b * (Tmax + 1) + s] = v;
    }
    if (bad && u == 0)
        flag(dev_status, TSD_DEV_BAD_TREE);
}

int launch_tree_mask(const int32_t *parent, const int32_t *n_nodes, int B, int Tmax,
                     uint32_t *mask, int32_t *depth, int32_t *first_child, int32_t *next_sibling,
                     int32_t *dev_status, cudaStream_t stream)
{
    if (B == 0)
        return TSD_OK;
    const int W = (Tmax + 31) / 32;
    tree_mask_kernel<<<B, kMaxTree, 0, stream>>>(parent, n_nodes, Tmax, W, mask, depth,
                                                 first_child, next_sibling, dev_status);
    TSD_LAUNCH_CHECK();
    return TSD_OK;
}

}  // namespace tsd
