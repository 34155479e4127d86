// Stochastic tree verification for callers that cannot allocate device memory.
//
// tsd_tree_verify_stochastic needs a small scratch area (the per-CTA partial
// sums its teams exchange and their barrier counters; its size does not
// depend on the problem).  Some callers have no way to
// provide one: a serving engine that has already handed nearly all device
// memory to its KV-cache pool, or code that reaches this library through a
// plain C interface with no device allocator of its own.  For them this file
// keeps that scratch in one fixed-size array in device memory that the
// library itself defines, so the call needs no cudaMalloc, no workspace and
// no allocating library routine.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it (kNoallocScratchBytes) until the process exits.  In host
// code its name only stands in for the symbol, so its device address is
// looked up once per device with cudaGetSymbolAddress while that device is
// current, and that address is what the kernels receive.
#include <mutex>

#include "tsd_common.cuh"

namespace {

constexpr size_t kNoallocScratchBytes = TSD_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_verify_scratch[kNoallocScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_verify_scratch on the current device (looked up on the
// first call made while that device is current, then cached).
int scratch_for_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        (void)cudaGetLastError();
        return TSD_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_verify_scratch) != cudaSuccess || p == nullptr) {
            (void)cudaGetLastError();
            return TSD_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return TSD_OK;
}

}  // namespace

extern "C" int tsd_tree_verify_stochastic_noalloc(
    const float *logits, double temperature, const float *q_probs, int Rq, const int32_t *q_row,
    const int32_t *tokens, const int32_t *n_nodes, const int32_t *first_child,
    const int32_t *next_sibling, const double *u_accept, const double *u_sample, int B, int Tmax,
    int V, int32_t *out_tokens, int32_t *out_path, int32_t *n_accepted, int32_t *dev_status,
    tsd_stream_t stream)
{
    TSD_NVTX_RANGE();
    if (B < 0 || Tmax < 1 || Tmax > TSD_MAX_TREE || V < 1 || Rq < 1 || !(temperature > 0.0))
        return TSD_ERR_SHAPE;
    if (B == 0)
        return TSD_OK;
    if (!logits || !q_probs || !q_row || !tokens || !n_nodes || !first_child || !next_sibling ||
        !u_accept || !u_sample || !out_tokens || !out_path || !n_accepted)
        return TSD_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(logits) & 15u) || (reinterpret_cast<uintptr_t>(q_probs) & 15u))
        return TSD_ERR_ALIGN;
    if (tsd::verify_stochastic_scratch() > kNoallocScratchBytes)
        return TSD_ERR_WORKSPACE;   // cannot happen with the constants above
    void *scratch = nullptr;
    const int rc = scratch_for_current_device(&scratch);
    if (rc != TSD_OK)
        return rc;
    // The launcher zeroes the team counters on the stream before the kernel;
    // every other scratch entry is written before it is read.
    return tsd::launch_verify_stochastic(logits, temperature, q_probs, Rq, q_row, tokens, n_nodes,
                                         first_child, next_sibling, u_accept, u_sample, B, Tmax,
                                         V, out_tokens, out_path, n_accepted, scratch, dev_status,
                                         reinterpret_cast<cudaStream_t>(stream));
}
