// Tree verification from the target model's logits (SpecInfer explainer,
// section "ツリー検証アルゴリズム").
//
// Both verifiers run in two launches:
//   1. a row kernel, one CTA per (logits row, sequence), for the rows whose
//      node has children (the root included).  Greedy: argmax of the row.
//      Stochastic: max, Z = sum exp((l-m)/T) in fp64, then multi-step
//      speculative sampling over the node's children in ascending index --
//      acceptance test u*q(x) <= p(x) with p(x) > 0, and after each rejection
//      the residual normaliser S = sum max(0, p - q) of the updated
//      distribution p <- max(0, p - q)/S.  Every internal node is decided in
//      parallel, whether or not the final path reaches it.
//   2. a finalize kernel, one CTA per sequence, that walks from the root
//      through the accepted children and emits the path, then the last token:
//      greedy -> argmax of the terminal row; stochastic -> inverse-CDF draw
//      from the terminal's (residual) distribution with a block-wide fp64
//      prefix scan.  A terminal that is a leaf gets its row statistics here.
//
// Residual distributions are never materialised: p^(i)(x) is recomputed per
// element from the logits row, the rejected siblings' q rows and their
// normalisers, with the same element-wise formula as the definition, so the
// only difference from a sequential fp64 evaluation is the summation order
// of Z, S and the cumulative sums.
#include <climits>

#include "tsd_common.cuh"

namespace tsd {

namespace {

constexpr int kRowThreads = 512;
constexpr int kWarps = kRowThreads / 32;

struct VerifyWs {
    int32_t *argmax;   // [B][Tmax+1]
    int32_t *accepted; // [B][Tmax+1]  accepted child per row, -1 none
    float *rmax;       // [B][Tmax+1]
    double *Z;         // [B][Tmax+1]
    double *S;         // [B][Tmax]    residual normaliser after rejecting child c
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

VerifyWs carve(void *ws, int B, int Tmax)
{
    const size_t R = (size_t)B * (Tmax + 1), N = (size_t)B * Tmax;
    char *p = static_cast<char *>(ws);
    VerifyWs w;
    w.Z = reinterpret_cast<double *>(p);
    p += align256(R * sizeof(double));
    w.S = reinterpret_cast<double *>(p);
    p += align256(N * sizeof(double));
    w.argmax = reinterpret_cast<int32_t *>(p);
    p += align256(R * sizeof(int32_t));
    w.accepted = reinterpret_cast<int32_t *>(p);
    p += align256(R * sizeof(int32_t));
    w.rmax = reinterpret_cast<float *>(p);
    return w;
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ bool better(float v, int i, float bv, int bi)
{
    return v > bv || (v == bv && i < bi);
}

__device__ void block_argmax(float &v, int &i, float *shv, int *shi)
{
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
        v = lane < kWarps ? shv[lane] : -INFINITY;
        i = lane < kWarps ? shi[lane] : INT_MAX;
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

__device__ int block_min_int(int v, int *sh)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0)
        sh[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < kWarps ? sh[lane] : INT_MAX;
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

__device__ int block_max_int(int v, int *sh)
{
    return -block_min_int(-v, sh);
}

// Row argmax (lowest index among the maxima), float4 loads when V % 4 == 0.
__device__ int row_argmax(const float *__restrict__ row, int V, float *shv, int *shi)
{
    float bv = -INFINITY;
    int bi = INT_MAX;
    if ((V & 3) == 0) {
        const float4 *r4 = reinterpret_cast<const float4 *>(row);
        for (int j = threadIdx.x; j < V / 4; j += kRowThreads) {
            const float4 x = __ldg(r4 + j);
            const int i0 = 4 * j;
            if (better(x.x, i0, bv, bi)) { bv = x.x; bi = i0; }
            if (better(x.y, i0 + 1, bv, bi)) { bv = x.y; bi = i0 + 1; }
            if (better(x.z, i0 + 2, bv, bi)) { bv = x.z; bi = i0 + 2; }
            if (better(x.w, i0 + 3, bv, bi)) { bv = x.w; bi = i0 + 3; }
        }
    } else {
        for (int j = threadIdx.x; j < V; j += kRowThreads) {
            const float x = __ldg(row + j);
            if (better(x, j, bv, bi)) { bv = x; bi = j; }
        }
    }
    block_argmax(bv, bi, shv, shi);
    return bi == INT_MAX ? 0 : bi;
}

__device__ float row_max(const float *__restrict__ row, int V, float *sh)
{
    float m = -INFINITY;
    if ((V & 3) == 0) {
        const float4 *r4 = reinterpret_cast<const float4 *>(row);
        for (int j = threadIdx.x; j < V / 4; j += kRowThreads) {
            const float4 x = __ldg(r4 + j);
            m = fmaxf(fmaxf(m, x.x), fmaxf(fmaxf(x.y, x.z), x.w));
        }
    } else {
        for (int j = threadIdx.x; j < V; j += kRowThreads)
            m = fmaxf(m, __ldg(row + j));
    }
    return block_max(m, sh);
}

// exp((l - m) / T) summed in fp64.
__device__ double row_Z(const float *__restrict__ row, int V, double m, double temp, double *sh)
{
    double z = 0.0;
    for (int j = threadIdx.x; j < V; j += kRowThreads)
        z += exp(((double)__ldg(row + j) - m) / temp);
    return block_sum(z, sh);
}

// Rejected siblings so far: their q rows and residual normalisers.
struct Residual {
    const float *q[kMaxTree];
    double S[kMaxTree];
    int n;
};

// p^(n)(x): the target distribution after the first n rejections.
__device__ __forceinline__ double residual_p(float lx, double m, double temp, double Z,
                                             const Residual &res, int x)
{
    double p = exp(((double)lx - m) / temp) / Z;
    for (int j = 0; j < res.n; ++j) {
        if (res.S[j] > 0.0) {
            const double r = p - (double)__ldg(res.q[j] + x);
            p = (r > 0.0 ? r : 0.0) / res.S[j];
        }
    }
    return p;
}

// sum_x max(0, p^(n)(x) - q(x))
__device__ double residual_mass(const float *__restrict__ row, const float *__restrict__ q, int V,
                                double m, double temp, double Z, const Residual &res,
                                double *sh)
{
    double s = 0.0;
    for (int x = threadIdx.x; x < V; x += kRowThreads) {
        const double r = residual_p(__ldg(row + x), m, temp, Z, res, x) - (double)__ldg(q + x);
        s += r > 0.0 ? r : 0.0;
    }
    return block_sum(s, sh);
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
    const int a = row_argmax(logits + ((size_t)b * (Tmax + 1) + r) * V, V, shv, shi);
    if (threadIdx.x == 0)
        argmax_ws[(size_t)b * (Tmax + 1) + r] = a;
}

__global__ void __launch_bounds__(kRowThreads)
    greedy_finalize_kernel(const float *__restrict__ logits, const int32_t *__restrict__ tokens,
                           const int32_t *__restrict__ parent,
                           const int32_t *__restrict__ n_nodes,
                           const uint32_t *__restrict__ mask,
                           const int32_t *__restrict__ first_child, int Tmax, int V,
                           const int32_t *__restrict__ argmax_ws, int32_t *__restrict__ out_tokens,
                           int32_t *__restrict__ out_path, int32_t *__restrict__ n_accepted,
                           int32_t *dev_status)
{
    __shared__ uint32_t matched[kMaskWords];
    __shared__ float shv[kWarps];
    __shared__ int shi[kWarps];
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
    key = block_max_int(key, shi);
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
        bonus = row_argmax(logits + ((size_t)b * (Tmax + 1) + row) * V, V, shv, shi);
    if (u == 0) {
        out_tokens[(size_t)b * (Tmax + 1) + n] = bonus;
        n_accepted[b] = n;
    }
}

// -------------------------------------------------------------- stochastic
__global__ void __launch_bounds__(kRowThreads)
    mss_rows_kernel(const float *__restrict__ logits, double temp,
                    const float *__restrict__ q_probs, int Rq, const int32_t *__restrict__ q_row,
                    const int32_t *__restrict__ tokens, const int32_t *__restrict__ n_nodes,
                    const int32_t *__restrict__ first_child,
                    const int32_t *__restrict__ next_sibling,
                    const double *__restrict__ u_accept, int Tmax, int V, VerifyWs ws)
{
    __shared__ float shf[kWarps];
    __shared__ double shd[kWarps];
    __shared__ Residual res;
    __shared__ int decision;
    const int r = blockIdx.x, b = blockIdx.y;
    int T;
    if (!sequence_ok(n_nodes, first_child, b, Tmax, T) || r > T)
        return;
    int c = first_child[(size_t)b * (Tmax + 1) + r];
    if (c < 0)
        return;
    const float *row = logits + ((size_t)b * (Tmax + 1) + r) * V;
    const float mf = row_max(row, V, shf);
    const double m = (double)mf;
    const double Z = row_Z(row, V, m, temp, shd);
    if (threadIdx.x == 0)
        res.n = 0;
    __syncthreads();
    int accepted = -1;
    while (c >= 0) {
        const int x = tokens[(size_t)b * Tmax + c];
        const int qr = q_row[(size_t)b * Tmax + c];
        if (x < 0 || x >= V || qr < 0 || qr >= Rq)
            break;   // malformed; the finalize kernel reports it
        const float *qc = q_probs + ((size_t)b * Rq + qr) * V;
        if (threadIdx.x == 0) {
            const double px = residual_p(row[x], m, temp, Z, res, x);
            const double qx = (double)qc[x];
            const double u = u_accept[(size_t)b * Tmax + c];
            decision = (px > 0.0 && u * qx <= px) ? 1 : 0;
        }
        __syncthreads();
        if (decision) {
            accepted = c;
            break;
        }
        const double S = residual_mass(row, qc, V, m, temp, Z, res, shd);
        if (threadIdx.x == 0) {
            res.q[res.n] = qc;
            res.S[res.n] = S;
            res.n += 1;
            ws.S[(size_t)b * Tmax + c] = S;
        }
        __syncthreads();
        c = next_sibling[(size_t)b * Tmax + c];
    }
    if (threadIdx.x == 0) {
        const size_t i = (size_t)b * (Tmax + 1) + r;
        ws.accepted[i] = accepted;
        ws.rmax[i] = mf;
        ws.Z[i] = Z;
    }
}

// Inverse-CDF draw from p^(n) over the row, fp64 block scan in tiles of
// 4 * kRowThreads consecutive tokens.
__device__ int residual_draw(const float *__restrict__ row, int V, double m, double temp, double Z,
                             const Residual &res, double u, double *shd, int *shi)
{
    __shared__ double warp_tot[kWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    double carry = 0.0;
    int last_pos = -1;
    for (int base = 0; base < V; base += 4 * kRowThreads) {
        const int x0 = base + 4 * threadIdx.x;
        double p[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int x = x0 + k;
            p[k] = x < V ? residual_p(__ldg(row + x), m, temp, Z, res, x) : 0.0;
            if (p[k] > 0.0)
                last_pos = x;
        }
        const double mine = ((p[0] + p[1]) + p[2]) + p[3];
        // inclusive warp scan of the per-thread sums
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
        for (int w2 = 0; w2 < kWarps; ++w2) {
            if (w2 < warp)
                wbase += warp_tot[w2];
            tile += warp_tot[w2];
        }
        double C = carry + wbase + (incl - mine);
        int found = INT_MAX;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            C += p[k];
            if (found == INT_MAX && x0 + k < V && C > u)
                found = x0 + k;
        }
        found = block_min_int(found, shi);
        if (found != INT_MAX)
            return found;
        carry += tile;
    }
    return block_max_int(last_pos, shi);
}

__global__ void __launch_bounds__(kRowThreads)
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
    __shared__ float shf[kWarps];
    __shared__ double shd[kWarps];
    __shared__ int shi[kWarps];
    __shared__ Residual res;
    __shared__ int term_row, n_path;
    const int b = blockIdx.x, u = threadIdx.x;
    int T;
    if (!sequence_ok(n_nodes, first_child, b, Tmax, T)) {
        if (u == 0)
            n_accepted[b] = -1;
        return;
    }
    int bad = 0;
    if (u < T) {
        const int x = tokens[(size_t)b * Tmax + u];
        const int qr = q_row[(size_t)b * Tmax + u];
        bad = (x < 0 || x >= V) ? TSD_DEV_BAD_TOKEN : 0;
        bad |= (qr < 0 || qr >= Rq) ? TSD_DEV_BAD_QROW : 0;
    }
    if (__syncthreads_or(bad)) {
        if (bad)
            flag(dev_status, bad);
        if (u == 0)
            n_accepted[b] = -1;
        return;
    }
    if (u == 0) {
        int row = 0, n = 0;
        while (n < T) {
            const int c = ws.accepted[(size_t)b * (Tmax + 1) + row];
            if (first_child[(size_t)b * (Tmax + 1) + row] < 0 || c < 0)
                break;
            out_path[(size_t)b * Tmax + n] = c;
            out_tokens[(size_t)b * (Tmax + 1) + n] = tokens[(size_t)b * Tmax + c];
            ++n;
            row = c + 1;
        }
        term_row = row;
        n_path = n;
        res.n = 0;
    }
    __syncthreads();
    const int row = term_row;
    const float *lrow = logits + ((size_t)b * (Tmax + 1) + row) * V;
    double m, Z;
    int c = first_child[(size_t)b * (Tmax + 1) + row];
    if (c >= 0) {
        // every child was rejected: statistics and normalisers from the row kernel
        m = (double)ws.rmax[(size_t)b * (Tmax + 1) + row];
        Z = ws.Z[(size_t)b * (Tmax + 1) + row];
        if (u == 0) {
            int n = 0;
            for (; c >= 0; c = next_sibling[(size_t)b * Tmax + c]) {
                res.q[n] = q_probs + ((size_t)b * Rq + q_row[(size_t)b * Tmax + c]) * V;
                res.S[n] = ws.S[(size_t)b * Tmax + c];
                ++n;
            }
            res.n = n;
        }
        __syncthreads();
    } else {
        m = (double)row_max(lrow, V, shf);
        Z = row_Z(lrow, V, m, temp, shd);
    }
    const double us = u_sample[(size_t)b * (Tmax + 1) + row];
    const int pick = residual_draw(lrow, V, m, temp, Z, res, us, shd, shi);
    if (u == 0) {
        out_tokens[(size_t)b * (Tmax + 1) + n_path] = pick;
        n_accepted[b] = n_path;
    }
}

}  // namespace

size_t verify_workspace(int B, int Tmax, int V)
{
    (void)V;
    const size_t R = (size_t)B * (Tmax + 1), N = (size_t)B * Tmax;
    return align256(R * sizeof(double)) + align256(N * sizeof(double)) +
           align256(R * sizeof(int32_t)) * 2 + align256(R * sizeof(float));
}

int launch_verify_greedy(const float *logits, const int32_t *tokens, const int32_t *parent,
                         const int32_t *n_nodes, const uint32_t *mask,
                         const int32_t *first_child, int B, int Tmax, int V,
                         int32_t *out_tokens, int32_t *out_path, int32_t *n_accepted, void *ws,
                         int32_t *dev_status, cudaStream_t stream)
{
    if (B == 0)
        return TSD_OK;
    const VerifyWs w = carve(ws, B, Tmax);
    greedy_rows_kernel<<<dim3(Tmax + 1, B), kRowThreads, 0, stream>>>(logits, n_nodes,
                                                                      first_child, Tmax, V,
                                                                      w.argmax);
    TSD_LAUNCH_CHECK();
    greedy_finalize_kernel<<<B, kRowThreads, 0, stream>>>(
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
    const VerifyWs w = carve(ws, B, Tmax);
    mss_rows_kernel<<<dim3(Tmax + 1, B), kRowThreads, 0, stream>>>(
        logits, temperature, q_probs, Rq, q_row, tokens, n_nodes, first_child, next_sibling,
        u_accept, Tmax, V, w);
    TSD_LAUNCH_CHECK();
    mss_finalize_kernel<<<B, kRowThreads, 0, stream>>>(
        logits, temperature, q_probs, Rq, q_row, tokens, n_nodes, first_child, next_sibling,
        u_sample, Tmax, V, w, out_tokens, out_path, n_accepted, dev_status);
    TSD_LAUNCH_CHECK();
    return TSD_OK;
}

}  // namespace tsd
