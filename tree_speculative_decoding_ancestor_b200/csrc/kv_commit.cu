// Commit of the accepted path (SpecInfer explainer, "Tree Attention のカーネル
// 融合", item 2: the tree's KV entries stay consistent with the existing KV
// cache; the flatkey.ai guide's verification diagram: the accepted prefix is
// committed).  After verification the K and V rows of the accepted nodes
// u_0 < u_1 < ... < u_{n-1} move from cache positions P_b + u_i to P_b + i,
// for every KV head, and the prefix grows to P_b + n.
//
// One CTA per (KV head, sequence).  A destination can be another accepted
// row's source (path [0, 2, 3]: position P+2 is read for i = 1 and written
// for i = 2), so the CTA first copies all n source rows of K and V into
// shared memory (16-byte vectors, every thread busy), waits for the whole
// CTA, and only then writes the destinations.  Rows already in place
// (u_i == i) are neither read nor written.  The path is checked before
// anything moves: entries strictly increasing, in [0, Tmax), and P + u < Lmax.
#include <atomic>

#include "tsd_common.cuh"

namespace tsd {

namespace {

constexpr int kCommitThreads = 256;

__global__ void __launch_bounds__(kCommitThreads)
    kv_commit_kernel(uint8_t *__restrict__ k, uint8_t *__restrict__ v,
                     const int32_t *__restrict__ prefix_len, const int32_t *__restrict__ out_path,
                     const int32_t *__restrict__ n_accepted, int Tmax, int Hkv, int Lmax,
                     int row_bytes, int32_t *__restrict__ new_prefix, int32_t *dev_status)
{
    extern __shared__ uint4 stage[];   // [2 (K, V)][n][row_bytes / 16]
    __shared__ int s_path[kMaxTree];
    const int h = blockIdx.x, b = blockIdx.y;
    const int n = n_accepted[b], P = prefix_len[b];
    if (n < 0) {   // malformed upstream (already reported there): nothing moves
        if (h == 0 && threadIdx.x == 0)
            new_prefix[b] = P;
        return;
    }
    bool ok = n <= Tmax && P >= 0;
    if (ok && (int)threadIdx.x < n)
        s_path[threadIdx.x] = out_path[(size_t)b * Tmax + threadIdx.x];
    __syncthreads();
    if (ok && (int)threadIdx.x < n) {
        const int i = threadIdx.x, u = s_path[i];
        ok = u >= 0 && u < Tmax && (i == 0 || u > s_path[i - 1]) && P + u < Lmax;
    }
    ok = __syncthreads_and(ok) != 0;
    if (h == 0 && threadIdx.x == 0) {
        new_prefix[b] = ok ? P + n : P;
        if (!ok)
            flag(dev_status, TSD_DEV_BAD_PATH);
    }
    if (!ok)
        return;
    const int vec = row_bytes / 16;
    const int total = n * vec;   // vectors per tensor
    const size_t plane = (size_t)Lmax * row_bytes;
    uint8_t *const kb = k + ((size_t)b * Hkv + h) * plane;
    uint8_t *const vb = v + ((size_t)b * Hkv + h) * plane;
    // extent of one (sequence, KV head) plane in 16-byte vectors
    const long long plane_vec = (long long)Lmax * vec;
    for (int idx = threadIdx.x; idx < 2 * total; idx += kCommitThreads) {
        const int t = idx >= total, r = idx - t * total, i = r / vec, c = r - i * vec;
        const int u = s_path[i];
        if (u != i && in_bounds((long long)(P + u) * vec + c, plane_vec, dev_status))
            stage[idx] = reinterpret_cast<const uint4 *>((t ? vb : kb) + (size_t)(P + u) * row_bytes)[c];
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < 2 * total; idx += kCommitThreads) {
        const int t = idx >= total, r = idx - t * total, i = r / vec, c = r - i * vec;
        if (s_path[i] != i && in_bounds((long long)(P + i) * vec + c, plane_vec, dev_status))
            reinterpret_cast<uint4 *>((t ? vb : kb) + (size_t)(P + i) * row_bytes)[c] = stage[idx];
    }
}

size_t kv_commit_smem(int Tmax, int row_bytes) { return (size_t)2 * Tmax * row_bytes; }

}  // namespace

int launch_kv_commit(void *k_cache, void *v_cache, const int32_t *prefix_len,
                     const int32_t *out_path, const int32_t *n_accepted, int B, int Tmax, int Hkv,
                     int Lmax, int row_bytes, int32_t *new_prefix, int32_t *dev_status,
                     cudaStream_t stream)
{
    if (B == 0)
        return TSD_OK;
    const size_t smem = kv_commit_smem(Tmax, row_bytes);
    if (smem > 48 * 1024) {
        // raise the kernel's limit once per device to the largest staging
        // buffer any shape can need (2 x TSD_MAX_TREE rows of 512 bytes)
        constexpr int kMaxDevices = 64;
        static std::atomic<bool> raised[kMaxDevices];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
            (void)cudaGetLastError();
            return TSD_ERR_CUDA;
        }
        if (!raised[dev].load()) {
            if (cudaFuncSetAttribute(kv_commit_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kv_commit_smem(kMaxTree, 512)) != cudaSuccess) {
                (void)cudaGetLastError();
                return TSD_ERR_CUDA;
            }
            raised[dev].store(true);
        }
    }
    kv_commit_kernel<<<dim3(Hkv, B), kCommitThreads, smem, stream>>>(
        static_cast<uint8_t *>(k_cache), static_cast<uint8_t *>(v_cache), prefix_len, out_path,
        n_accepted, Tmax, Hkv, Lmax, row_bytes, new_prefix, dev_status);
    TSD_LAUNCH_CHECK();
    return TSD_OK;
}

}  // namespace tsd
