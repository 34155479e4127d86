// Tree attention on CUDA cores (warp-shuffle FMA path).
//
// Computes, for every node u < T_b and query head h,
//   out[b][u][h] = softmax_j(scale * q . k_j) v_j  over j in S_u
// (SpecInfer explainer, "トークンツリー構造の仕組み", the Attention(Q_u,
// K_{S_u}, V_{S_u}) equation), where S_u is the committed prefix plus the
// tree positions whose bit is set in the ancestor mask.
//
// This path serves fp32 inputs and query blocks too small for the tensor
// cores to pay.  Query rows of one KV head are packed GQA-style as
// r = u * G + g (G = Hq / Hkv), 16 rows per CTA, 4 rows per warp.  Keys are
// streamed through shared memory in tiles of 32 (lane j owns key j for the
// score, lane l owns dims l, l+32, ... for the output); the softmax is the
// online (running max / running sum) form in the log2 domain.  Long key
// ranges are split across CTAs (split-KV) and merged by combine_kernel with
// the usual log-sum-exp rescaling.
#include <cfloat>

#include <algorithm>
#include <cstdlib>

#include "tsd_common.cuh"

namespace tsd {

namespace {

constexpr int kSimtThreads = 128;
constexpr int kSimtRows = 16;     // query rows per CTA (4 warps x 4 rows)
constexpr int kSimtKeys = 32;     // keys per shared-memory tile
constexpr float kLog2e = 1.4426950408889634f;

struct SimtPlan {
    int row_chunks;   // ceil(Tmax * G / kSimtRows)
    int nsplit;       // key-range splits
    int keys_per_split;
};

SimtPlan simt_plan(const AttnArgs &a, int num_sms)
{
    SimtPlan p;
    const int G = a.Hq / a.Hkv;
    p.row_chunks = (a.Tmax * G + kSimtRows - 1) / kSimtRows;
    const long base = (long)p.row_chunks * a.B * a.Hkv;
    const int max_split = (a.Lmax + 127) / 128;   // at least 128 keys per split
    int ns = (int)((2L * num_sms + base - 1) / (base > 0 ? base : 1));
    ns = ns < 1 ? 1 : ns;
    ns = ns > max_split ? max_split : ns;
    ns = ns > 64 ? 64 : ns;
    if (const char *e = std::getenv("TSD_ATTN_SPLITS")) {   // forced split count
        const int n = std::atoi(e);
        if (n >= 1)
            ns = std::min(std::min(n, 64), max_split);
    }
    p.nsplit = ns;
    int kps = (a.Lmax + ns - 1) / ns;
    p.keys_per_split = (kps + kSimtKeys - 1) / kSimtKeys * kSimtKeys;
    return p;
}

template <typename Elt, int D>
__global__ void __launch_bounds__(kSimtThreads)
    tree_attn_simt_kernel(const Elt *__restrict__ q, const Elt *__restrict__ kc,
                          const Elt *__restrict__ vc, const int32_t *__restrict__ prefix_len,
                          const int32_t *__restrict__ n_nodes, const uint32_t *__restrict__ mask,
                          int Tmax, int Hq, int Hkv, int Lmax, int W, float scale_log2,
                          int keys_per_split, int nsplit, Elt *__restrict__ out,
                          float *__restrict__ part_o, float2 *__restrict__ part_ml,
                          int32_t *dev_status, KvPages pages)
{
    constexpr int DL = D / 32;
    __shared__ float sq[kSimtRows][D];
    __shared__ float sk[kSimtKeys][D + 1];
    __shared__ float sv[kSimtKeys][D];
    __shared__ uint32_t smask[kSimtRows][kMaskWords];

    const int chunk = blockIdx.x;
    const int bkv = blockIdx.y;
    const int split = blockIdx.z;
    const int b = bkv / Hkv, hk = bkv % Hkv;
    const int G = Hq / Hkv;
    const int T = n_nodes[b];
    const int P = prefix_len[b];
    if (!tree_header_ok(T, Tmax) || P < 0 || P + T > Lmax) {
        if (chunk == 0 && split == 0 && hk == 0 && threadIdx.x == 0)
            flag(dev_status, TSD_DEV_BAD_PREFIX);
        return;
    }
    const int R = T * G;
    const int row0 = chunk * kSimtRows;
    if (row0 >= R)
        return;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int k_begin = split * keys_per_split;
    const int k_end = min(k_begin + keys_per_split, P + T);

    // extents of the buffers (checked build)
    const int B = gridDim.y / Hkv;
    const long long n_rows = (long long)B * Tmax * Hq;          // q / out rows
    const long long n_kv = kv_rows_total(pages, B, Hkv, Lmax);   // K / V rows
    // Stage this CTA's query rows and their ancestor masks.
    for (int i = threadIdx.x; i < kSimtRows * D; i += kSimtThreads) {
        const int lr = i / D, d = i % D, r = row0 + lr;
        float x = 0.f;
        if (r < R) {
            const int u = r / G, h = hk * G + r % G;
            if (in_bounds(((long long)b * Tmax + u) * Hq + h, n_rows, dev_status))
                x = to_float(q[(((size_t)b * Tmax + u) * Hq + h) * D + d]);
        }
        sq[lr][d] = x;
    }
    for (int i = threadIdx.x; i < kSimtRows * kMaskWords; i += kSimtThreads) {
        const int lr = i / kMaskWords, w = i % kMaskWords, r = row0 + lr;
        const long long mi = ((long long)b * Tmax + r / G) * W + w;
        smask[lr][w] = (r < R && w < W && in_bounds(mi, (long long)B * Tmax * W, dev_status))
                           ? mask[mi] : 0u;
    }

    float o[4][DL];
    float m[4], l[4];
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        m[rr] = -INFINITY;
        l[rr] = 0.f;
#pragma unroll
        for (int i = 0; i < DL; ++i)
            o[rr][i] = 0.f;
    }

    for (int kt = k_begin; kt < k_end; kt += kSimtKeys) {
        __syncthreads();
        for (int i = threadIdx.x; i < kSimtKeys * D; i += kSimtThreads) {
            const int j = i / D, d = i % D, pos = kt + j;
            float kx = 0.f, vx = 0.f;
            if (pos < k_end) {
                const long long row = kv_row(pages, b, hk, Hkv, Lmax, pos);
                if (row >= 0 && in_bounds(row, n_kv, dev_status)) {
                    kx = to_float(kc[row * D + d]);
                    vx = to_float(vc[row * D + d]);
                } else if (d == 0) {
                    flag(dev_status, TSD_DEV_BAD_PAGE);   // that key reads as zero
                }
            }
            sk[j][d] = kx;
            sv[j][d] = vx;
        }
        __syncthreads();
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
            const int lr = warp * 4 + rr;
            if (row0 + lr >= R)
                continue;   // warp-uniform
            const int pos = kt + lane;
            bool valid = pos < k_end;
            if (valid && pos >= P) {
                const int v = pos - P;
                valid = (smask[lr][v >> 5] >> (v & 31)) & 1u;
            }
            float s = 0.f;
#pragma unroll 16
            for (int d = 0; d < D; ++d)
                s = fmaf(sq[lr][d], sk[lane][d], s);
            s = valid ? s * scale_log2 : -INFINITY;
            const float m_new = fmaxf(m[rr], warp_max(s));
            if (m_new == -INFINITY)
                continue;   // nothing visible yet (warp-uniform)
            const float p = valid ? exp2f(s - m_new) : 0.f;
            const float alpha = exp2f(m[rr] - m_new);
            l[rr] = l[rr] * alpha + warp_sum(p);
#pragma unroll
            for (int i = 0; i < DL; ++i)
                o[rr][i] *= alpha;
#pragma unroll 8
            for (int j = 0; j < kSimtKeys; ++j) {
                const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
                for (int i = 0; i < DL; ++i)
                    o[rr][i] = fmaf(pj, sv[j][lane + 32 * i], o[rr][i]);
            }
            m[rr] = m_new;
        }
    }

#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const int r = row0 + warp * 4 + rr;
        if (r >= R)
            continue;
        const int u = r / G, h = hk * G + r % G;
        const size_t row = ((size_t)b * Tmax + u) * Hq + h;
        if (!in_bounds((long long)row, n_rows, dev_status))
            continue;
        if (nsplit == 1) {
            const float inv = l[rr] > 0.f ? 1.f / l[rr] : 0.f;   // a row with no key: 0
#pragma unroll
            for (int i = 0; i < DL; ++i)
                out[row * D + lane + 32 * i] = from_float<Elt>(o[rr][i] * inv);
        } else {
            const size_t prow = (size_t)split * ((size_t)gridDim.y / Hkv * Tmax * Hq) + row;
#pragma unroll
            for (int i = 0; i < DL; ++i)
                part_o[prow * D + lane + 32 * i] = o[rr][i];
            if (lane == 0)
                part_ml[prow] = make_float2(m[rr], l[rr]);
        }
    }
}

// Merge split-KV partials (log2-domain running max m, sum l, unnormalised o).
template <typename Elt, int D>
__global__ void __launch_bounds__(256)
    combine_kernel(const float *__restrict__ part_o, const float2 *__restrict__ part_ml,
                   int nsplit, const int32_t *__restrict__ prefix_len,
                   const int32_t *__restrict__ n_nodes, int B, int Tmax, int Hq, int Lmax,
                   Elt *__restrict__ out)
{
    constexpr int DL = D / 32;
    const int lane = threadIdx.x & 31;
    const size_t nrows = (size_t)B * Tmax * Hq;
    const size_t row = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= nrows)
        return;
    const int b = (int)(row / ((size_t)Tmax * Hq));
    const int u = (int)((row / Hq) % Tmax);
    if (!in_bounds(b, B, nullptr))
        return;
    const int T = n_nodes[b], P = prefix_len[b];
    if (!tree_header_ok(T, Tmax) || P < 0 || P + T > Lmax || u >= T)
        return;
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) {
        const float2 ml = part_ml[(size_t)s * nrows + row];
        if (ml.y > 0.f)
            M = fmaxf(M, ml.x);
    }
    float acc[DL];
#pragma unroll
    for (int i = 0; i < DL; ++i)
        acc[i] = 0.f;
    float L = 0.f;
    for (int s = 0; s < nsplit; ++s) {
        const float2 ml = part_ml[(size_t)s * nrows + row];
        if (!(ml.y > 0.f))
            continue;
        const float w = exp2f(ml.x - M);
        L += w * ml.y;
#pragma unroll
        for (int i = 0; i < DL; ++i)
            acc[i] = fmaf(w, part_o[((size_t)s * nrows + row) * D + lane + 32 * i], acc[i]);
    }
    // a row that no split saw a key for (a caller mask without the node's own
    // bit and no prefix) is written as zeros, as the single-split paths do
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int i = 0; i < DL; ++i)
        out[row * D + lane + 32 * i] = from_float<Elt>(acc[i] * inv);
}

// Splits that see no key of a row still have to publish an empty partial.
__global__ void clear_partials_kernel(float2 *part_ml, size_t n)
{
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x)
        part_ml[i] = make_float2(-INFINITY, 0.f);
}

template <typename Elt, int D>
int launch_typed(const AttnArgs &a, const SimtPlan &p, void *ws, cudaStream_t stream)
{
    const size_t nrows = (size_t)a.B * a.Tmax * a.Hq;
    float *part_o = nullptr;
    float2 *part_ml = nullptr;
    if (p.nsplit > 1) {
        part_ml = reinterpret_cast<float2 *>(ws);
        part_o = reinterpret_cast<float *>(static_cast<char *>(ws) +
                                           (((size_t)p.nsplit * nrows * sizeof(float2) + 255) &
                                            ~(size_t)255));
        clear_partials_kernel<<<256, 256, 0, stream>>>(part_ml, (size_t)p.nsplit * nrows);
        TSD_LAUNCH_CHECK();
    }
    dim3 grid(p.row_chunks, a.B * a.Hkv, p.nsplit);
    const float scale_log2 = a.scale * kLog2e;
    tree_attn_simt_kernel<Elt, D><<<grid, kSimtThreads, 0, stream>>>(
        static_cast<const Elt *>(a.q), static_cast<const Elt *>(a.k), static_cast<const Elt *>(a.v),
        a.prefix_len, a.n_nodes, a.mask, a.Tmax, a.Hq, a.Hkv, a.Lmax, (a.Tmax + 31) / 32,
        scale_log2, p.keys_per_split, p.nsplit, static_cast<Elt *>(a.out), part_o, part_ml,
        a.dev_status, a.pages);
    TSD_LAUNCH_CHECK();
    if (p.nsplit > 1) {
        const unsigned blocks = (unsigned)((nrows + 7) / 8);
        combine_kernel<Elt, D><<<blocks, 256, 0, stream>>>(part_o, part_ml, p.nsplit,
                                                         a.prefix_len, a.n_nodes, a.B, a.Tmax,
                                                         a.Hq, a.Lmax, static_cast<Elt *>(a.out));
        TSD_LAUNCH_CHECK();
    }
    return TSD_OK;
}

template <int D>
int combine_typed(int dtype, const float *part_o, const float2 *part_ml, int nsplit,
                  const int32_t *prefix_len, const int32_t *n_nodes, int B, int Tmax, int Hq,
                  int Lmax, void *out, cudaStream_t stream)
{
    const size_t nrows = (size_t)B * Tmax * Hq;
    const unsigned blocks = (unsigned)((nrows + 7) / 8);
    if (dtype == TSD_F32)
        combine_kernel<float, D><<<blocks, 256, 0, stream>>>(
            part_o, part_ml, nsplit, prefix_len, n_nodes, B, Tmax, Hq, Lmax,
            static_cast<float *>(out));
    else
        combine_kernel<__nv_bfloat16, D><<<blocks, 256, 0, stream>>>(
            part_o, part_ml, nsplit, prefix_len, n_nodes, B, Tmax, Hq, Lmax,
            static_cast<__nv_bfloat16 *>(out));
    return TSD_OK;
}

}  // namespace

// Shared with the tensor-core path: empty partials, and the split-KV merge.
// The caller checks and counts the launch.
void launch_clear_partials(float2 *part_ml, size_t n, cudaStream_t stream)
{
    clear_partials_kernel<<<256, 256, 0, stream>>>(part_ml, n);
}

int launch_combine(int dtype, int D, const float *part_o, const float2 *part_ml, int nsplit,
                   const int32_t *prefix_len, const int32_t *n_nodes, int B, int Tmax, int Hq,
                   int Lmax, void *out, cudaStream_t stream)
{
    if (D == 64)
        return combine_typed<64>(dtype, part_o, part_ml, nsplit, prefix_len, n_nodes, B, Tmax,
                                 Hq, Lmax, out, stream);
    if (D == 128)
        return combine_typed<128>(dtype, part_o, part_ml, nsplit, prefix_len, n_nodes, B, Tmax,
                                  Hq, Lmax, out, stream);
    return TSD_ERR_DTYPE;
}

void simt_attention_plan(const AttnArgs &a, int num_sms, int32_t out[4])
{
    const SimtPlan p = simt_plan(a, num_sms);
    out[0] = TSD_PLAN_SIMT;
    out[1] = p.row_chunks;
    out[2] = p.nsplit;
    out[3] = p.keys_per_split;
}

size_t simt_attention_workspace(const AttnArgs &a, int num_sms)
{
    const SimtPlan p = simt_plan(a, num_sms);
    if (p.nsplit <= 1)
        return 0;
    const size_t nrows = (size_t)a.B * a.Tmax * a.Hq;
    const size_t ml = ((size_t)p.nsplit * nrows * sizeof(float2) + 255) & ~(size_t)255;
    return ml + (size_t)p.nsplit * nrows * a.D * sizeof(float);
}

int launch_simt_attention(const AttnArgs &a, void *ws, size_t ws_bytes, int num_sms,
                          cudaStream_t stream)
{
    const SimtPlan p = simt_plan(a, num_sms);
    if (ws_bytes < simt_attention_workspace(a, num_sms))
        return TSD_ERR_WORKSPACE;
    if (a.dtype == TSD_F32) {
        if (a.D == 64)
            return launch_typed<float, 64>(a, p, ws, stream);
        if (a.D == 128)
            return launch_typed<float, 128>(a, p, ws, stream);
    } else {
        if (a.D == 64)
            return launch_typed<__nv_bfloat16, 64>(a, p, ws, stream);
        if (a.D == 128)
            return launch_typed<__nv_bfloat16, 128>(a, p, ws, stream);
    }
    return TSD_ERR_DTYPE;
}

}  // namespace tsd
