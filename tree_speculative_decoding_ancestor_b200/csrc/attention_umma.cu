// Tree attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Computes the same result as the CUDA-core path (SpecInfer explainer,
// "トークンツリー構造の仕組み": softmax(Q_u K_{S_u}^T / sqrt(d_k)) V_{S_u},
// S_u = committed prefix + the node's ancestors-or-self) for bf16 inputs with
// head_dim 128.
//
// Work unit = (row block, (b, KV head), KV split).  The query rows of one KV
// head are packed GQA-style, r = u * G + g, so a 128-row block is a dense
// [128 x 128] A operand no matter how the tree and the head group split it.
// Per key tile of 128 positions:
//     S   = Q K^T           tcgen05.mma, A = Q (smem), B = K tile (smem, TMA),
//                           fp32 accumulator in TMEM (two S buffers ping-pong)
//     P   = 2^(S*scale*log2e - m)   softmax warps: TMEM -> registers, ancestor
//                           mask (only on the tiles that reach the tree), online
//                           max/sum, P packed to bf16 and stored back into the
//                           S buffer's TMEM columns
//     O  += P V             tcgen05.mma with A = P read from TMEM and B = the V
//                           tile (smem, MN-major), O accumulated in TMEM
// The running max is only raised (and O rescaled) when a tile's max exceeds it
// by more than 2^8, which keeps O rescales rare while P stays < 256.
//
// Warp roles (192 threads): warp 0 issues TMA loads of K and V into two
// separate rings, warp 1 owns TMEM and issues the MMAs (one elected lane),
// warps 2-5 run the softmax, one query row per thread (TMEM lane = row).
// Every mbarrier wait is bounded: after ~2 s it raises a CTA-wide abort flag,
// reports TSD_DEV_TIMEOUT and the CTA unwinds, frees its TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "sm100_ptx.cuh"
#include "tsd_common.cuh"

namespace tsd {

void launch_clear_partials(float2 *part_ml, size_t n, cudaStream_t stream);
int launch_combine(int dtype, int D, const float *part_o, const float2 *part_ml, int nsplit,
                   const int32_t *prefix_len, const int32_t *n_nodes, int B, int Tmax, int Hq,
                   int Lmax, void *out, cudaStream_t stream);

namespace {

constexpr int BM = 128;        // query rows per CTA
constexpr int BN = 128;        // keys per tile
constexpr int HD = 128;        // head dim
constexpr int NSK = 3;         // K ring stages
constexpr int NSV = 2;         // V ring stages
constexpr int kThreads = 192;  // 6 warps
constexpr uint32_t kSub = BN * 128;          // [128 rows][64 bf16] sub-tile, 16 KB
constexpr uint32_t kTile = 2 * kSub;         // [128][128] bf16, 32 KB
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTile;
constexpr uint32_t kOffV = kOffK + NSK * kTile;
constexpr uint32_t kOffBar = kOffV + NSV * kTile;
constexpr int kNumBars = 1 + 2 * NSK + 2 * NSV + 2 + 2 + 1;
constexpr uint32_t kOffMisc = kOffBar + 8 * kNumBars;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;   // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

// mbarrier addresses: q_full, k_full[NSK], k_empty[NSK], v_full[NSV],
// v_empty[NSV], s_full[2], p_full[2], o_ready -- consecutive 8-byte words.
struct Bars {
    uint32_t base;
    __device__ uint32_t q_full() const { return base; }
    __device__ uint32_t k_full(int s) const { return base + 8u * (1 + s); }
    __device__ uint32_t k_empty(int s) const { return base + 8u * (1 + NSK + s); }
    __device__ uint32_t v_full(int s) const { return base + 8u * (1 + 2 * NSK + s); }
    __device__ uint32_t v_empty(int s) const { return base + 8u * (1 + 2 * NSK + NSV + s); }
    __device__ uint32_t s_full(int i) const { return base + 8u * (1 + 2 * NSK + 2 * NSV + i); }
    __device__ uint32_t p_full(int i) const { return base + 8u * (3 + 2 * NSK + 2 * NSV + i); }
    __device__ uint32_t o_ready() const { return base + 8u * (5 + 2 * NSK + 2 * NSV); }
};

// A wait whose outcome is the same on every lane of the warp (the TMEM
// loads/stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort)
{
    const bool ok = ptx::mbar_wait(bar, parity, abort);
    return __all_sync(0xffffffffu, ok);
}

// K-major, 128-byte-swizzled operand made of two [rows][64] sub-tiles: the
// descriptor for the kk-th 16-wide slice of the 128-wide contraction dim.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int kk)
{
    const uint32_t addr = tile + (uint32_t)(kk >> 2) * kSub + (uint32_t)(kk & 3) * 32u;
    return ptx::smem_desc_sw128(addr, 16u, 1024u);
}

// V tile as the MN-major B operand of O += P V: the kk-th group of 16 keys;
// the two 64-wide halves of head_dim are kSub bytes apart.
__device__ __forceinline__ uint64_t desc_v(uint32_t tile, int kk)
{
    return ptx::smem_desc_sw128(tile + (uint32_t)kk * 16u * 128u, kSub, 1024u);
}

__device__ __forceinline__ uint32_t mask_word(const uint32_t (&mw)[4], int v)
{
    return v < 32 ? mw[0] : v < 64 ? mw[1] : v < 96 ? mw[2] : mw[3];
}

__global__ void __launch_bounds__(kThreads, 1)
    tree_attn_umma_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __nv_bfloat16 *__restrict__ q,
                          const int32_t *__restrict__ prefix_len,
                          const int32_t *__restrict__ n_nodes, const uint32_t *__restrict__ mask,
                          int Tmax, int Hq, int Hkv, int Lmax, int W, float scale_log2,
                          int keys_per_split, int nsplit, __nv_bfloat16 *__restrict__ out,
                          float *__restrict__ part_o, float2 *__restrict__ part_ml,
                          int32_t *dev_status)
{
    extern __shared__ uint8_t smem_raw[];
    const int rb = blockIdx.x, pair = blockIdx.y, split = blockIdx.z;
    const int b = pair / Hkv, hk = pair % Hkv;
    const int G = Hq / Hkv;
    const int T = n_nodes[b], P = prefix_len[b];
    if (!tree_header_ok(T, Tmax) || P < 0 || P + T > Lmax) {
        if (rb == 0 && split == 0 && hk == 0 && threadIdx.x == 0)
            flag(dev_status, TSD_DEV_BAD_PREFIX);
        return;
    }
    const int R = T * G;
    const int kb = split * keys_per_split;
    const int ke = min(kb + keys_per_split, P + T);
    if (rb * BM >= R || kb >= ke)
        return;   // no rows or no keys: the partials stay empty
    const int ntiles = (ke - kb + BN - 1) / BN;

    // 1024-byte aligned carve-up (128-byte swizzle atoms repeat every 1024 B).
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t sQ = base + kOffQ, sK = base + kOffK, sV = base + kOffV;
    const Bars bars{base + kOffBar};
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(gbase + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        ptx::mbar_init(bars.q_full(), 128);
        for (int i = 0; i < NSK; ++i) {
            ptx::mbar_init(bars.k_full(i), 1);
            ptx::mbar_init(bars.k_empty(i), 1);
        }
        for (int i = 0; i < NSV; ++i) {
            ptx::mbar_init(bars.v_full(i), 1);
            ptx::mbar_init(bars.v_empty(i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bars.s_full(i), 1);
            ptx::mbar_init(bars.p_full(i), 128);
        }
        ptx::mbar_init(bars.o_ready(), 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_addr((const void *)tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            ptx::prefetch_tmap(&tmK);
            ptx::prefetch_tmap(&tmV);
            const int z = b * Hkv + hk;
            // Order of consumption by the MMA warp: K0, K1, V0, K2, V1, ...
            for (int i = 0; i <= ntiles; ++i) {
                if (i < ntiles) {
                    const int s = i % NSK;
                    if (i >= NSK &&
                        !ptx::mbar_wait(bars.k_empty(s), ((i / NSK) - 1) & 1, abort_flag))
                        break;
                    ptx::mbar_arrive_expect_tx(bars.k_full(s), kTile);
                    const uint32_t dst = sK + s * kTile;
                    const int pos = kb + i * BN;
                    ptx::tma_load_3d(dst, &tmK, 0, pos, z, bars.k_full(s));
                    ptx::tma_load_3d(dst + kSub, &tmK, 64, pos, z, bars.k_full(s));
                }
                if (i >= 1) {
                    const int j = i - 1, s = j % NSV;
                    if (j >= NSV &&
                        !ptx::mbar_wait(bars.v_empty(s), ((j / NSV) - 1) & 1, abort_flag))
                        break;
                    ptx::mbar_arrive_expect_tx(bars.v_full(s), kTile);
                    const uint32_t dst = sV + s * kTile;
                    const int pos = kb + j * BN;
                    ptx::tma_load_3d(dst, &tmV, 0, pos, z, bars.v_full(s));
                    ptx::tma_load_3d(dst + kSub, &tmV, 64, pos, z, bars.v_full(s));
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idesc_qk = ptx::idesc_bf16(BM, BN, false, false);
        constexpr uint32_t idesc_pv = ptx::idesc_bf16(BM, HD, false, true);
        bool ok = warp_wait(bars.q_full(), 0, abort_flag);
        ptx::tc_fence_after();
        for (int i = 0; ok && i <= ntiles; ++i) {
            if (i < ntiles) {
                const int s = i % NSK, sb = i & 1;
                if (!warp_wait(bars.k_full(s), (i / NSK) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                if (lane == 0) {
                    const uint32_t d = tmem + (sb ? kColS1 : kColS0);
#pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk)
                        ptx::mma_ss(d, desc_kmajor(sQ, kk), desc_kmajor(sK + s * kTile, kk),
                                    idesc_qk, kk > 0 ? 1u : 0u);
                    ptx::mma_commit(bars.s_full(sb));
                    ptx::mma_commit(bars.k_empty(s));
                }
                __syncwarp();
            }
            if (i >= 1) {
                const int j = i - 1, pb = j & 1, s = j % NSV;
                if (!warp_wait(bars.p_full(pb), (j >> 1) & 1, abort_flag) ||
                    !warp_wait(bars.v_full(s), (j / NSV) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                // Cache rows at or beyond P + T may hold anything (NaN included):
                // zero them so that P = 0 there contributes exactly nothing.
                const int first_bad = P + T - (kb + j * BN);
                if (first_bad < BN) {
                    uint8_t *vt = gbase + (sV - base) + s * kTile;
                    for (int row = max(first_bad, 0) + (lane >> 3); row < BN; row += 4) {
                        const int c = lane & 7;
                        *reinterpret_cast<uint4 *>(vt + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4 *>(vt + kSub + row * 128 + c * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                }
                if (lane == 0) {
                    const uint32_t a = tmem + (pb ? kColS1 : kColS0);
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        ptx::mma_ts(tmem + kColO, a + kk * 8, desc_v(sV + s * kTile, kk), idesc_pv,
                                    (j > 0 || kk > 0) ? 1u : 0u);
                    ptx::mma_commit(bars.v_empty(s));
                    ptx::mma_commit(bars.o_ready());
                }
                __syncwarp();
            }
        }
    } else {
        // ------------------------------------------------ softmax warps 2..5
        const int quarter = warp & 3;
        const int t = quarter * 32 + lane;   // row within the block == TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int r = rb * BM + t;
        const bool row_ok = r < R;
        const int u = row_ok ? r / G : 0;
        const int h = hk * G + (row_ok ? r % G : 0);

        // Q row -> shared memory in the 128-byte swizzled K-major layout.
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(
                q + (((size_t)b * Tmax + u) * Hq + h) * HD);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint4 x = row_ok ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
                const int sub = c >> 3, cc = c & 7;
                *reinterpret_cast<uint4 *>(gbase + kOffQ + sub * kSub + t * 128 +
                                           ((cc ^ (t & 7)) * 16)) = x;
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(bars.q_full());
        }
        uint32_t mw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int w = 0; w < 4; ++w)
            if (row_ok && w < W)
                mw[w] = mask[((size_t)b * Tmax + u) * W + w];

        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            const int sb = j & 1;
            const uint32_t scol = sb ? kColS1 : kColS0;
            if (!warp_wait(bars.s_full(sb), (j >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                ptx::tmem_ld32(tmem + lane_off + scol + c * 32, sr[c]);
            ptx::tmem_wait_ld();

            // Raw scores (masked ones -inf); the softmax scale (> 0) is applied
            // inside the exponent's FMA, and to the max once.
            const int pos0 = kb + j * BN;
            float s[BN];
            if (pos0 + BN <= min(P, ke)) {
#pragma unroll
                for (int k = 0; k < BN; ++k)
                    s[k] = __uint_as_float(sr[k >> 5][k & 31]);
            } else {
#pragma unroll
                for (int k = 0; k < BN; ++k) {
                    const int pos = pos0 + k;
                    bool valid = pos < ke;
                    if (valid && pos >= P) {
                        const int v = pos - P;
                        valid = (mask_word(mw, v) >> (v & 31)) & 1u;
                    }
                    s[k] = valid ? __uint_as_float(sr[k >> 5][k & 31]) : -INFINITY;
                }
            }
            // Tile max with 8 independent partial maxima (short dependency chains).
            float mx[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mx[i] = s[i];
#pragma unroll
            for (int k = 8; k < BN; ++k)
                mx[k & 7] = fmaxf(mx[k & 7], s[k]);
            const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                             scale_log2;
            const bool need = mt > m_run + kRescaleThreshold;   // false if mt is -inf
            const float m_new = need ? mt : m_run;
            const float alpha = need ? ptx::ex2(m_run - m_new) : 1.f;   // 0 when m_run = -inf
            if (__any_sync(0xffffffffu, need) && j > 0) {
                // O holds PV_0..PV_{j-1}: wait for the last of them, then rescale.
                if (!warp_wait(bars.o_ready(), (j - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    ptx::tmem_ld32(tmem + lane_off + kColO + c * 32, o);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                    ptx::tmem_st32(tmem + lane_off + kColO + c * 32, o);
                }
                ptx::tmem_wait_st();
            }
            l_run *= alpha;
            m_run = m_new;
            const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
            float lsum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t pk[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const float p0 = ptx::ex2(fmaf(s[c * 64 + 2 * k], scale_log2, neg_m));
                    const float p1 = ptx::ex2(fmaf(s[c * 64 + 2 * k + 1], scale_log2, neg_m));
                    lsum[k & 3] += p0 + p1;
                    pk[k] = ptx::pack_bf16(p0, p1);
                }
                ptx::tmem_st32(tmem + lane_off + scol + c * 32, pk);
            }
            ptx::tmem_wait_st();
            l_run += (lsum[0] + lsum[1]) + (lsum[2] + lsum[3]);
            ptx::tc_fence_before();
            ptx::mbar_arrive(bars.p_full(sb));
        }

        // ------------------------------------------------ epilogue
        if (ok && warp_wait(bars.o_ready(), (ntiles - 1) & 1, abort_flag)) {
            ptx::tc_fence_after();
            const size_t row = ((size_t)b * Tmax + u) * Hq + h;
            const size_t nrows = (size_t)gridDim.y / Hkv * Tmax * Hq;
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(tmem + lane_off + kColO + c * 32, o);
                ptx::tmem_wait_ld();
                if (!row_ok)
                    continue;
                if (nsplit == 1) {
                    uint4 *dst = reinterpret_cast<uint4 *>(out + row * HD + c * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 x;
                        x.x = ptx::pack_bf16(__uint_as_float(o[8 * v + 0]) * inv,
                                             __uint_as_float(o[8 * v + 1]) * inv);
                        x.y = ptx::pack_bf16(__uint_as_float(o[8 * v + 2]) * inv,
                                             __uint_as_float(o[8 * v + 3]) * inv);
                        x.z = ptx::pack_bf16(__uint_as_float(o[8 * v + 4]) * inv,
                                             __uint_as_float(o[8 * v + 5]) * inv);
                        x.w = ptx::pack_bf16(__uint_as_float(o[8 * v + 6]) * inv,
                                             __uint_as_float(o[8 * v + 7]) * inv);
                        dst[v] = x;
                    }
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(
                        part_o + ((size_t)split * nrows + row) * HD + c * 32);
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        dst[v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                             __uint_as_float(o[4 * v + 2]),
                                             __uint_as_float(o[4 * v + 3]));
                }
            }
            if (row_ok && nsplit > 1)
                part_ml[(size_t)split * nrows + row] = make_float2(m_run, l_run);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0)
        flag(dev_status, TSD_DEV_TIMEOUT);
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host
struct UmmaPlan {
    int nrb, nsplit, keys_per_split;
};

UmmaPlan umma_plan(const AttnArgs &a, int num_sms)
{
    UmmaPlan p;
    const int G = a.Hq / a.Hkv;
    p.nrb = (a.Tmax * G + BM - 1) / BM;
    const long base = (long)p.nrb * a.B * a.Hkv;
    const int tiles = (a.Lmax + BN - 1) / BN;
    int best = 1;
    double best_cost = 1e30;
    for (int ns = 1; ns <= 64 && ns <= tiles; ++ns) {
        const long units = base * ns;
        const long waves = (units + num_sms - 1) / num_sms;
        const int per = (tiles + ns - 1) / ns;
        const double cost = (double)waves * (per + 2);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = ns;
        }
    }
    p.nsplit = best;
    p.keys_per_split = ((tiles + best - 1) / best) * BN;
    return p;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [B*Hkv][Lmax][128] bf16 cache viewed as a 3-D tensor, boxes of [1][128][64].
bool make_kv_map(CUtensorMap *m, const void *ptr, int Lmax, int BH)
{
    auto fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)Lmax, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)Lmax * HD * 2};
    cuuint32_t box[3] = {64, BN, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool umma_attention_supported(const AttnArgs &a)
{
    // bf16, head_dim 128, and a packed query block large enough to feed the
    // tensor cores (smaller blocks stay on the CUDA-core path).
    return a.dtype == TSD_BF16 && a.D == HD && a.Tmax * (a.Hq / a.Hkv) >= 8;
}

size_t umma_attention_workspace(const AttnArgs &a, int num_sms)
{
    const UmmaPlan p = umma_plan(a, num_sms);
    if (p.nsplit <= 1)
        return 0;
    const size_t nrows = (size_t)a.B * a.Tmax * a.Hq;
    const size_t ml = ((size_t)p.nsplit * nrows * sizeof(float2) + 255) & ~(size_t)255;
    return ml + (size_t)p.nsplit * nrows * HD * sizeof(float);
}

int launch_umma_attention(const AttnArgs &a, void *ws, size_t ws_bytes, int num_sms,
                          cudaStream_t stream)
{
    const UmmaPlan p = umma_plan(a, num_sms);
    if (ws_bytes < umma_attention_workspace(a, num_sms))
        return TSD_ERR_WORKSPACE;
    CUtensorMap tmK, tmV;
    if (!make_kv_map(&tmK, a.k, a.Lmax, a.B * a.Hkv) ||
        !make_kv_map(&tmV, a.v, a.Lmax, a.B * a.Hkv))
        return TSD_ERR_CUDA;
    static bool attr_set = false;
    if (!attr_set) {
        TSD_CUDA_TRY(cudaFuncSetAttribute(tree_attn_umma_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)kSmemBytes));
        attr_set = true;
    }
    const size_t nrows = (size_t)a.B * a.Tmax * a.Hq;
    float *part_o = nullptr;
    float2 *part_ml = nullptr;
    if (p.nsplit > 1) {
        part_ml = reinterpret_cast<float2 *>(ws);
        part_o = reinterpret_cast<float *>(
            static_cast<char *>(ws) +
            (((size_t)p.nsplit * nrows * sizeof(float2) + 255) & ~(size_t)255));
        launch_clear_partials(part_ml, (size_t)p.nsplit * nrows, stream);
        TSD_LAUNCH_CHECK();
    }
    dim3 grid(p.nrb, a.B * a.Hkv, p.nsplit);
    tree_attn_umma_kernel<<<grid, kThreads, kSmemBytes, stream>>>(
        tmK, tmV, static_cast<const __nv_bfloat16 *>(a.q), a.prefix_len, a.n_nodes, a.mask,
        a.Tmax, a.Hq, a.Hkv, a.Lmax, (a.Tmax + 31) / 32, a.scale * kLog2e, p.keys_per_split,
        p.nsplit, static_cast<__nv_bfloat16 *>(a.out), part_o, part_ml, a.dev_status);
    TSD_LAUNCH_CHECK();
    if (p.nsplit > 1) {
        const int rc = launch_combine(a.dtype, a.D, part_o, part_ml, p.nsplit, a.prefix_len,
                                      a.n_nodes, a.B, a.Tmax, a.Hq, a.Lmax, a.out, stream);
        if (rc != TSD_OK)
            return rc;
        TSD_LAUNCH_CHECK();
    }
    return TSD_OK;
}

}  // namespace tsd
