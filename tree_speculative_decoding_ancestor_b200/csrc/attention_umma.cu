// Tree attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Computes the same result as the CUDA-core path (SpecInfer explainer,
// "トークンツリー構造の仕組み": softmax(Q_u K_{S_u}^T / sqrt(d_k)) V_{S_u},
// S_u = committed prefix + the node's ancestors-or-self) for bf16 inputs with
// head_dim 128.
//
// The query rows of one KV head are packed GQA-style, r = u * G + g, so a
// block of 128 rows is one dense [128 x 128] A operand however the tree and
// the head group divide it.  Per key tile of 128 positions:
//     S   = Q K^T      tcgen05.mma, A = Q (smem), B = K tile (smem, TMA),
//                      fp32 accumulator in TMEM
//     P   = 2^(S*scale*log2e - m)   softmax warps: TMEM -> registers, ancestor
//                      mask only on tiles that reach the tree (one 32-bit
//                      visibility word per 32 keys), online max/sum, P packed
//                      to bf16 and written back over the S columns
//     O  += P V        tcgen05.mma with A = P from TMEM, B = V tile (MN-major)
// The running max is only raised (O rescaled in TMEM) when a tile exceeds it
// by more than 2^8, so rescales are rare while P stays below 256.  The
// softmax issues few instructions per score (packed fp32x2 scaling and sums,
// three-input max); with one softmax warp per SM sub-partition it is bound
// by that warp's issue rate.  Cache rows at or beyond P_b + T_b are zeroed
// in shared memory before the PV product, so garbage there (NaN included)
// never leaks.  One mbarrier arrival per softmax warp (not per thread).
//
// Two kernels share this machinery:
//   * tree_attn_rows_kernel: one CTA per (128-row block, (b, KV head), KV
//     split); 6 warps -- TMA producer, MMA issuer, 4 softmax warps; TMEM
//     holds NS score buffers (the scores of the next key tiles are ready
//     while the softmax works) and O.  Two instances: 128-key tiles with
//     three S buffers at one CTA per SM (more than 128 packed rows), and
//     64-key tiles with two S buffers at two CTAs per SM (at most 128 packed
//     rows, where the KV stream is the bound: two co-resident CTAs keep
//     twice the loads in flight and hide each other's prologue and tail).
//   * tree_attn_keysplit_kernel (at most 128 rows; selected with
//     TSD_ATTN_SMALL_VARIANT=keysplit): one CTA per ((b, KV head), split);
//     two 4-warp softmax groups take the even and odd key tiles of the same
//     query tile, each with its own S and O in TMEM, and their (O, m, l) are
//     merged by log-sum-exp at the end.
// K and V stream through separate TMA rings (128-byte swizzle).  Every
// mbarrier wait is bounded: after ~2 s it raises a CTA-wide abort flag, the
// CTA reports TSD_DEV_TIMEOUT, unwinds, frees its TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "sm100_ptx.cuh"
#include "tsd_common.cuh"

namespace tsd {

void launch_clear_partials(float2 *part_ml, size_t n, cudaStream_t stream);
int launch_combine(int dtype, int D, const float *part_o, const float2 *part_ml, int nsplit,
                   const int32_t *prefix_len, const int32_t *n_nodes, int B, int Tmax, int Hq,
                   int Lmax, void *out, cudaStream_t stream);

namespace {

constexpr int BQ = 128;        // query rows per tile
constexpr int HD = 128;        // head dim
constexpr uint32_t kSubQ = BQ * 128;         // Q [128 rows][64 bf16] sub-tile, 16 KB
constexpr uint32_t kTileQ = 2 * kSubQ;       // Q tile [128][128] bf16, 32 KB
constexpr uint32_t kOffQ = 0;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr float kLazyLimit = 18446744073709551616.0f;   // 2^64: headroom of a P tile sum
constexpr int kTableCache = 1024;   // block-table entries of a CTA's key range kept in smem

// Tile geometry of a kernel: keys per tile, K and V ring stages, TMEM
// columns; shared memory holds Q, the K ring, the V ring, the mbarriers.
template <int BN_, int NSK_, int NSV_, uint32_t TMEM_COLS>
struct Geo {
    static constexpr int BN = BN_;                       // keys per tile
    static constexpr int NSK = NSK_;                     // K ring stages
    static constexpr int NSV = NSV_;                     // V ring stages
    static constexpr uint32_t kSub = BN * 128;           // [BN rows][64 bf16] sub-tile
    static constexpr uint32_t kTile = 2 * kSub;          // [BN][128] bf16
    static constexpr uint32_t kOffK = kOffQ + kTileQ;
    static constexpr uint32_t kOffV = kOffK + NSK * kTile;
    static constexpr uint32_t kOffBar = kOffV + NSV * kTile;
    static constexpr int kNumBars = 1 + 2 * NSK + 2 * NSV + 16;
    static constexpr uint32_t kOffMisc = kOffBar + 8 * kNumBars;
    static constexpr uint32_t kOffXchg = kOffMisc + 16;    // the softmax pairs' exchange slots
    static constexpr uint32_t kXchgBytes = 4 * 528;        // 4 x sizeof(PairXchg)
    static constexpr uint32_t kOffTable = kOffXchg + kXchgBytes;   // paged: block-table slice
    static constexpr uint32_t kSmemBytes = kOffTable + 4 * kTableCache + 1024;   // + alignment slack
    static constexpr uint32_t kTmemCols = TMEM_COLS;
};
// 128-key tiles, 197 KB of shared memory and all 512 TMEM columns: one CTA
// per SM (rows and key-split kernels).
using Wide = Geo<128, 3, 2, 512>;
// 64-key tiles, 97 KB and 256 columns: two CTAs per SM (paired rows kernel).
using Half = Geo<64, 2, 2, 256>;
static_assert(Wide::kSmemBytes <= 232448, "shared memory budget");
static_assert(2 * (Half::kSmemBytes + 1024) <= 233472, "two CTAs per SM");

constexpr int kSplitThreads = 384;      // key-split kernel: 12 warps

// mbarrier addresses: q_full, k_full[NSK], k_empty[NSK], v_full[NSV],
// v_empty[NSV], s_full[4], p_full[4], o_ready[4], pair[4] -- consecutive
// 8-byte words.
template <class Gm>
struct Bars {
    static constexpr int NSK = Gm::NSK, NSV = Gm::NSV;
    uint32_t base;
    __device__ uint32_t q_full() const { return base; }
    __device__ uint32_t k_full(int s) const { return base + 8u * (1 + s); }
    __device__ uint32_t k_empty(int s) const { return base + 8u * (1 + NSK + s); }
    __device__ uint32_t v_full(int s) const { return base + 8u * (1 + 2 * NSK + s); }
    __device__ uint32_t v_empty(int s) const { return base + 8u * (1 + 2 * NSK + NSV + s); }
    __device__ uint32_t s_full(int i) const { return base + 8u * (1 + 2 * NSK + 2 * NSV + i); }
    __device__ uint32_t p_full(int i) const { return base + 8u * (5 + 2 * NSK + 2 * NSV + i); }
    __device__ uint32_t o_ready(int i) const { return base + 8u * (9 + 2 * NSK + 2 * NSV + i); }
    // the two softmax warps of TMEM lane quarter i meet here (two arrivals)
    __device__ uint32_t pair(int i) const { return base + 8u * (13 + 2 * NSK + 2 * NSV + i); }
};

// A wait whose outcome is the same on every lane of the warp (the TMEM
// loads/stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort)
{
    const bool ok = ptx::mbar_wait(bar, parity, abort);
    return __all_sync(0xffffffffu, ok);
}

// warp_wait for a phase that this warp already tested with ptx::mbar_test
// (`tested`, this lane's result) while it did other work: when every lane
// saw the phase complete the wait costs one vote.  The test must have been
// issued after the phase before it completed (else a stale phase passes).
__device__ __forceinline__ bool warp_wait_tested(uint32_t tested, uint32_t bar, uint32_t parity,
                                                 volatile int *abort)
{
    if (__all_sync(0xffffffffu, tested != 0u))
        return true;
    return warp_wait(bar, parity, abort);
}

// One arrival per warp: the lanes' prior writes (TMEM stores after their
// wait::st and fence, or shared-memory stores after their proxy fence) are
// ordered before lane 0's arrival by the warp barrier.
__device__ __forceinline__ void warp_arrive(uint32_t bar)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0)
        ptx::mbar_arrive(bar);
}

// K-major, 128-byte-swizzled operand made of two [rows][64] sub-tiles `sub`
// bytes apart: the descriptor for the 16-wide slice kk of the 128-wide
// contraction dim is the base descriptor plus slice_off(kk, sub) (the
// address field is addr >> 4 and shared addresses stay below 256 KB, so
// adding to the packed word never carries out of it).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile)
{
    return ptx::smem_desc_sw128(tile, 16u, 1024u);
}
__device__ __forceinline__ uint64_t slice_off(int kk, uint32_t sub)
{
    return ((uint32_t)(kk >> 2) * sub + (uint32_t)(kk & 3) * 32u) >> 4;
}

// V tile as the MN-major B operand of O += P V (group kk of 16 keys at
// + kk * 2 KB); the two 64-wide halves of head_dim are `sub` bytes apart.
__device__ __forceinline__ uint64_t desc_v(uint32_t tile, uint32_t sub)
{
    return ptx::smem_desc_sw128(tile, sub, 1024u);
}

__device__ __forceinline__ uint32_t mask_word(const uint32_t (&mw)[4], int v)
{
    return v < 32 ? mw[0] : v < 64 ? mw[1] : v < 96 ? mw[2] : mw[3];
}

// Visibility of the 32 keys pos0 .. pos0 + 31 for one query row: bit k is set
// iff key pos0 + k is below ke and is either a prefix position (< P) or a
// tree node on the row's root path (bit pos0 + k - P of the ancestor mask).
__device__ __forceinline__ uint32_t valid_bits(int pos0, int P, int ke, const uint32_t (&mw)[4])
{
    auto low_ones = [](int n) -> uint32_t {
        return n >= 32 ? 0xffffffffu : (n <= 0 ? 0u : ((1u << n) - 1u));
    };
    const uint32_t prefix = low_ones(P - pos0);
    const int lo = pos0 - P;   // ancestor-mask bit of key pos0
    uint32_t tree = 0u;
    if (lo >= 0 && lo < 128) {
        const int w = lo >> 5, sh = lo & 31;
        const uint32_t a = mask_word(mw, w * 32);
        const uint32_t c = w < 3 ? mask_word(mw, w * 32 + 32) : 0u;
        tree = sh ? (a >> sh) | (c << (32 - sh)) : a;
    } else if (lo < 0 && lo > -32) {
        tree = mw[0] << (-lo);
    }
    return (prefix | tree) & low_ones(ke - pos0);
}

// Per-CTA set-up shared by both kernels: 1024-byte aligned carve-up of the
// dynamic shared memory, barrier initialisation, TMEM allocation (warp 1).
template <class Gm>
struct Setup {
    uint8_t *gbase;
    uint32_t base, sQ, sK, sV, tmem;
    Bars<Gm> bars;
    volatile int *abort_flag;
};

template <class Gm>
__device__ __forceinline__ Setup<Gm> cta_setup(uint8_t *smem_raw, uint32_t q_arrivals,
                                               uint32_t p_arrivals)
{
    constexpr int NSK = Gm::NSK, NSV = Gm::NSV;
    constexpr uint32_t kOffMisc = Gm::kOffMisc;
    Setup<Gm> su;
    const uint32_t raw = ptx::smem_addr(smem_raw);
    su.base = (raw + 1023u) & ~1023u;
    su.gbase = smem_raw + (su.base - raw);
    su.sQ = su.base + kOffQ;
    su.sK = su.base + Gm::kOffK;
    su.sV = su.base + Gm::kOffV;
    su.bars = Bars<Gm>{su.base + Gm::kOffBar};
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(su.gbase + kOffMisc);
    su.abort_flag = reinterpret_cast<volatile int *>(su.gbase + kOffMisc + 4);
    if (threadIdx.x == 0) {
        ptx::mbar_init(su.bars.q_full(), q_arrivals);
        for (int i = 0; i < NSK; ++i) {
            ptx::mbar_init(su.bars.k_full(i), 1);
            ptx::mbar_init(su.bars.k_empty(i), 1);
        }
        for (int i = 0; i < NSV; ++i) {
            ptx::mbar_init(su.bars.v_full(i), 1);
            ptx::mbar_init(su.bars.v_empty(i), 1);
        }
        for (int i = 0; i < 4; ++i) {
            ptx::mbar_init(su.bars.s_full(i), 1);
            ptx::mbar_init(su.bars.o_ready(i), 1);
            ptx::mbar_init(su.bars.p_full(i), p_arrivals);
            ptx::mbar_init(su.bars.pair(i), 2);
        }
        *su.abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::fence_proxy_async_smem();
    }
    if ((threadIdx.x >> 5) == 1) {
        ptx::tmem_alloc(ptx::smem_addr((const void *)tmem_slot), Gm::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    su.tmem = *tmem_slot;
    return su;
}

template <class Gm>
__device__ __forceinline__ void cta_teardown(const Setup<Gm> &su, int32_t *dev_status)
{
    ptx::tc_fence_before();
    __syncthreads();
    if (*su.abort_flag && threadIdx.x == 0)
        flag(dev_status, TSD_DEV_TIMEOUT);
    if ((threadIdx.x >> 5) == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(su.tmem, Gm::kTmemCols);
    }
}

// The TMA loads of one [BN keys][128] K or V tile starting at logical key
// position pos0 into `dst` (two 64-column halves).  Contiguous cache: one box
// per half at (x, pos0, b * Hkv + hk).  Paged cache: one box per page the
// tile touches (box rows = min(BN, page_size); a box never straddles a page
// since both are powers of two and pos0 is a multiple of BN) at (x, row in
// page, page * Hkv + hk).  A box that starts at or beyond the sequence's end
// loads any valid page: those keys are masked and their V rows zeroed.
// The block-table entries of the pages a CTA's key range [kb, seq_end)
// touches, staged in shared memory by the producer warp before its first
// load (at most kTableCache of them; entries past that are read from global
// memory), so that a ring slot's reload does not wait for a global load.
struct PageCache {
    const int32_t *sm;   // entries blk0 .. blk0 + n - 1
    int blk0, n;
};

template <class Gm>
__device__ __forceinline__ PageCache stage_pages(const Setup<Gm> &su, const KvPages &pages, int b,
                                                 int kb, int seq_end, int lane)
{
    PageCache pc{reinterpret_cast<const int32_t *>(su.gbase + Gm::kOffTable), 0, 0};
    if (!pages.table || seq_end <= kb)
        return pc;
    pc.blk0 = kb >> pages.log2_page;
    pc.n = min(((seq_end - 1) >> pages.log2_page) - pc.blk0 + 1, kTableCache);
    int32_t *dst = reinterpret_cast<int32_t *>(su.gbase + Gm::kOffTable);
    for (int i = lane; i < pc.n; i += 32)
        dst[i] = pages.table[(size_t)b * pages.max_blocks + pc.blk0 + i];
    __syncwarp();
    return pc;
}

template <class Gm>
__device__ __forceinline__ void load_kv_tile(uint32_t dst, const CUtensorMap *tm, uint32_t bar,
                                             int pos0, int b, int hk, int Hkv,
                                             const KvPages &pages, const PageCache &pc,
                                             int seq_end, int32_t *dev_status)
{
    if (!pages.table) {
        ptx::tma_load_3d(dst, tm, 0, pos0, b * Hkv + hk, bar);
        ptx::tma_load_3d(dst + Gm::kSub, tm, 64, pos0, b * Hkv + hk, bar);
        return;
    }
    const int rows = min(Gm::BN, pages.page_size);
    for (int r0 = 0; r0 < Gm::BN; r0 += rows) {
        const int pos = pos0 + r0;
        int z = hk, y = 0;
        if (pos < seq_end) {
            const int blk = pos >> pages.log2_page, ci = blk - pc.blk0;
            const int page = (ci >= 0 && ci < pc.n)
                                 ? pc.sm[ci]
                                 : pages.table[(size_t)b * pages.max_blocks + blk];
            if (page < 0 || page >= pages.num_pages)
                flag(dev_status, TSD_DEV_BAD_PAGE);   // page 0 stands in
            else
                z = page * Hkv + hk;
            y = pos & (pages.page_size - 1);
        }
        ptx::tma_load_3d(dst + r0 * 128, tm, 0, y, z, bar);
        ptx::tma_load_3d(dst + Gm::kSub + r0 * 128, tm, 64, y, z, bar);
    }
}

// TMA producer (one lane).  Load order: K_0 .. K_{NSK-1} and V_0 .. V_{NSV-1}
// into the empty rings, then ... V_m, K_{m+L}, V_{m+1}, ... with L = NSK +
// LA - NSV, LA the MMA warp's QK lookahead (QK_{j+LA} is issued right after
// PV_j).  A ring slot is reused once the product that read it is complete,
// so V_m's slot frees with PV_{m-NSV} and K_{m+L}'s with QK_{m+L-NSK}, the
// QK issued right after that same PV: each reload is issued as soon as its
// slot is free, a K tile has about LA tile periods to land, and no V reload
// queues behind a K reload gated one product later.  Deadlock-free: the
// product a K wait needs reads V tiles below m only, and the one a V wait
// needs reads K tiles below the K index already issued.  NS_PROD = 0: the
// MMA warp commits every product to the rings' own empty barriers as well.
// NS_PROD = NS (the number of score buffers, equal to the K ring's depth):
// the producer waits on the products' own barriers instead -- QK_{i-NSK}
// completes on s_full[i % NS], PV_{j-NSV} on o_ready[(j - NSV) % NS] --
// which saves the MMA thread two commits per tile.  Either wait names a phase
// that cannot be stale or ahead: the phase before it was waited for by the
// previous reload of the same ring slot, and the phase after it needs K_i
// (or V_{j+1}), which this producer has not loaded yet.
template <class Gm, int NS_PROD>
__device__ __forceinline__ void produce_kv(const Setup<Gm> &su, const CUtensorMap *tmK,
                                           const CUtensorMap *tmV, int b, int hk, int Hkv,
                                           int kb, int ntiles, const KvPages &pages,
                                           const PageCache &pc, int seq_end,
                                           int32_t *dev_status)
{
    constexpr int NSK = Gm::NSK, NSV = Gm::NSV, BN = Gm::BN;
    constexpr uint32_t kTile = Gm::kTile;
    static_assert(NS_PROD == 0 || NS_PROD == NSK, "score buffers and K ring in step");
    // the QK lookahead: NS for the rows kernels, 2 for the key-split kernel
    constexpr int kLead = NSK + (NS_PROD ? NS_PROD : 2) - NSV;
    ptx::prefetch_tmap(tmK);
    ptx::prefetch_tmap(tmV);
    int i = 0, j = 0;   // next K tile, next V tile
    while (i < ntiles || j < ntiles) {
        const bool take_k =
            i < ntiles && (j >= ntiles || i < NSK || (j >= NSV && i <= j - 1 + kLead));
        if (take_k) {
            const int s = i % NSK;
            const uint32_t k_free = NS_PROD ? su.bars.s_full(s) : su.bars.k_empty(s);
            if (i >= NSK && !ptx::mbar_wait(k_free, ((i / NSK) - 1) & 1, su.abort_flag))
                break;
            ptx::mbar_arrive_expect_tx(su.bars.k_full(s), kTile);
            load_kv_tile<Gm>(su.sK + s * kTile, tmK, su.bars.k_full(s), kb + i * BN, b, hk, Hkv,
                             pages, pc, seq_end, dev_status);
            ++i;
        } else {
            const int s = j % NSV;
            if (j >= NSV) {
                const int r = j - NSV;   // PV_r read this slot last
                constexpr int NSP = NS_PROD ? NS_PROD : 1;
                // PV_r done: o_ready[r % NS] phase r / NS, or the ring's own
                // v_empty (which the MMA warp then commits as well)
                const bool ok =
                    !NS_PROD
                        ? ptx::mbar_wait(su.bars.v_empty(s), ((j / NSV) - 1) & 1, su.abort_flag)
                        : ptx::mbar_wait(su.bars.o_ready(r % NSP), (r / NSP) & 1,
                                         su.abort_flag);
                if (!ok)
                    break;
            }
            ptx::mbar_arrive_expect_tx(su.bars.v_full(s), kTile);
            load_kv_tile<Gm>(su.sV + s * kTile, tmV, su.bars.v_full(s), kb + j * BN, b, hk, Hkv,
                             pages, pc, seq_end, dev_status);
            ++j;
        }
    }
}

// MMA warp, S = Q K^T for key tile `t` into TMEM columns `col_s`.
template <class Gm, bool RING_COMMIT = true, bool COMMIT = true, bool WARP = true>
__device__ __forceinline__ void issue_qk(const Setup<Gm> &su, int lane, uint32_t col_s, int t,
                                         uint32_t s_full)
{
    constexpr uint32_t idesc = ptx::idesc_bf16(BQ, Gm::BN, false, false);
    const int st = t % Gm::NSK;
    if (lane == 0) {
        const uint64_t dq = desc_kmajor(su.sQ), dk = desc_kmajor(su.sK + st * Gm::kTile);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
            ptx::mma_ss(su.tmem + col_s, dq + slice_off(kk, kSubQ), dk + slice_off(kk, Gm::kSub),
                        idesc, kk > 0 ? 1u : 0u);
        if (COMMIT)
            ptx::mma_commit(s_full);
        if (COMMIT && RING_COMMIT)
            ptx::mma_commit(su.bars.k_empty(st));
    }
    if (WARP)
        __syncwarp();
}

// MMA warp, O += P V for key tile `t` (P in TMEM columns col_p); zeroes the
// V rows at or beyond P_b + T_b first.  P_SPLIT: the packed P of keys
// 64 .. 127 sits 64 columns after that of keys 0 .. 63 (each softmax half
// writes into its own score columns) instead of right after it.
// Zero the rows first_bad .. BN-1 of V ring slot vs (cache rows at or beyond
// P_b + T_b: masked keys whose P is 0, but 0 * NaN would not be), by one warp,
// then make the generic-proxy stores visible to the tensor cores.
template <class Gm>
__device__ __forceinline__ void zero_v_rows(const Setup<Gm> &su, int vs, int first_bad, int lane)
{
    uint8_t *vt = su.gbase + Gm::kOffV + vs * Gm::kTile;
    for (int row = max(first_bad, 0) + (lane >> 3); row < Gm::BN; row += 4) {
        const int c = lane & 7;
        *reinterpret_cast<uint4 *>(vt + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(vt + Gm::kSub + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
    }
    ptx::fence_proxy_async_smem();
    __syncwarp();
}

template <class Gm, bool RING_COMMIT = true, bool P_SPLIT = false, bool COMMIT = true,
          bool ZERO = true>
__device__ __forceinline__ void issue_pv(const Setup<Gm> &su, int lane, uint32_t col_p,
                                         uint32_t col_o, int t, bool accumulate, int first_bad,
                                         uint32_t o_ready)
{
    constexpr int BN = Gm::BN;
    constexpr uint32_t idesc = ptx::idesc_bf16(BQ, HD, false, true);
    const int vs = t % Gm::NSV;
    if (ZERO && first_bad < BN)
        zero_v_rows<Gm>(su, vs, first_bad, lane);
    ptx::tc_fence_after();
    if (lane == 0) {
        const uint64_t dv = desc_v(su.sV + vs * Gm::kTile, Gm::kSub);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t pc = P_SPLIT ? (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8)
                                        : (uint32_t)(kk * 8);
            ptx::mma_ts(su.tmem + col_o, su.tmem + col_p + pc,
                        dv + (uint64_t)((kk * 16u * 128u) >> 4), idesc,
                        (accumulate || kk > 0) ? 1u : 0u);
        }
        if (COMMIT && RING_COMMIT)
            ptx::mma_commit(su.bars.v_empty(vs));
        if (COMMIT)
            ptx::mma_commit(o_ready);
    }
    if (ZERO)
        __syncwarp();
}

// Softmax-warp helpers.  Row state of one query row of a tile.
struct RowCtx {
    int P, ke;
    uint32_t mw[4];
    float scale_log2;
};

// Q row `t` of the tile -> shared memory, 128-byte swizzled K-major layout;
// with SW = 2 warps per row, half hf loads the 64 dims hf*64 .. hf*64 + 63.
template <class Gm, int SW = 1>
__device__ __forceinline__ void load_q_row(const Setup<Gm> &su, const __nv_bfloat16 *__restrict__ q,
                                           bool row_ok, size_t q_off, int t, int hf = 0)
{
    uint8_t *dst = su.gbase + kOffQ;
    const uint4 *src = reinterpret_cast<const uint4 *>(q + q_off);
#pragma unroll
    for (int c = (SW == 2 ? hf * 8 : 0); c < (SW == 2 ? hf * 8 + 8 : 16); ++c) {
        const uint4 x = row_ok ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
        const int sub = c >> 3, cc = c & 7;
        *reinterpret_cast<uint4 *>(dst + sub * kSubQ + t * 128 + ((cc ^ (t & 7)) * 16)) = x;
    }
    ptx::fence_proxy_async_smem();
}

// Rescale this row's O (TMEM columns col_o) by alpha.
__device__ __forceinline__ void rescale_o(uint32_t taddr_o, float alpha)
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        ptx::tmem_ld32(taddr_o + c * 32, o);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k)
            o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
        ptx::tmem_st32(taddr_o + c * 32, o);
    }
    ptx::tmem_wait_st();
}

// P = 2^(s * scale - m) for 64 scores (two 32-column chunks already loaded
// and masked), packed to bf16 into pk[32]; returns their sum.  The scaling
// and the sums run on packed fp32 pairs, the exponentials on MUFU.
__device__ __forceinline__ float exp_pack64(const uint32_t (&sa)[32], const uint32_t (&sb)[32],
                                            float scale_log2, float neg_m, uint32_t (&pk)[32])
{
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        float x0, x1, x2, x3;
        ptx::fma2_bc(x0, x1, __uint_as_float(sa[2 * k]), __uint_as_float(sa[2 * k + 1]),
                     scale_log2, neg_m);
        ptx::fma2_bc(x2, x3, __uint_as_float(sb[2 * k]), __uint_as_float(sb[2 * k + 1]),
                     scale_log2, neg_m);
        const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1), p2 = ptx::ex2(x2), p3 = ptx::ex2(x3);
        const int a = (k & 1) * 2;
        ptx::add2(acc[a], acc[a + 1], p0, p1);
        ptx::add2(acc[a], acc[a + 1], p2, p3);
        pk[k] = ptx::pack_bf16(p0, p1);
        pk[16 + k] = ptx::pack_bf16(p2, p3);
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// P for 32 scores (one 32-column chunk, loaded and masked), packed to bf16
// into pk[16]; returns their sum.
__device__ __forceinline__ float exp_pack32(const uint32_t (&sa)[32], float scale_log2,
                                            float neg_m, uint32_t (&pk)[16])
{
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        float x0, x1;
        ptx::fma2_bc(x0, x1, __uint_as_float(sa[2 * k]), __uint_as_float(sa[2 * k + 1]),
                     scale_log2, neg_m);
        const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
        const int a = (k & 1) * 2;
        ptx::add2(acc[a], acc[a + 1], p0, p1);
        pk[k] = ptx::pack_bf16(p0, p1);
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

__device__ __forceinline__ void mask32(uint32_t (&s)[32], uint32_t bits)
{
#pragma unroll
    for (int k = 0; k < 32; ++k)
        s[k] = ((bits >> k) & 1u) ? s[k] : __float_as_uint(-INFINITY);
}

// Running maxima of 64 scores, 16 independent chains of 3-input maxima.
__device__ __forceinline__ void max32x2(const uint32_t (&sa)[32], const uint32_t (&sb)[32],
                                        float (&mx)[16])
{
#pragma unroll
    for (int k = 0; k < 32; ++k)
        mx[k & 15] = ptx::max3(mx[k & 15], __uint_as_float(sa[k]), __uint_as_float(sb[k]));
}

__device__ __forceinline__ float max16(const float (&mx)[16])
{
    float a = ptx::max3(mx[0], mx[1], mx[2]), b = ptx::max3(mx[3], mx[4], mx[5]);
    float c = ptx::max3(mx[6], mx[7], mx[8]), d = ptx::max3(mx[9], mx[10], mx[11]);
    float e = ptx::max3(mx[12], mx[13], mx[14]);
    return ptx::max3(ptx::max3(a, b, c), ptx::max3(d, e, mx[15]), -INFINITY);
}

// Online-softmax step for one tile whose scores sit in TMEM columns col_s:
// max, (rare) rescale of O, P over the S columns, running sum.  `wait_o`
// waits for the previous PV product when O must be rescaled.  Returns false
// on abort.
template <typename WaitO>
__device__ __forceinline__ bool softmax_tile(uint32_t taddr_s, uint32_t taddr_o, int pos0,
                                             const RowCtx &rc, bool first, float &m_run,
                                             float &l_run, WaitO wait_o)
{
    const bool masked = !(pos0 + Wide::BN <= min(rc.P, rc.ke));
    // max over the raw scores (scale > 0 is applied once), two chunks at a time
    float mx[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        mx[i] = -INFINITY;
#pragma unroll 1
    for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t sa[32], sb[32];
        ptx::tmem_ld32(taddr_s + c2 * 64, sa);
        ptx::tmem_ld32(taddr_s + c2 * 64 + 32, sb);
        ptx::tmem_wait_ld();
        if (masked) {
            mask32(sa, valid_bits(pos0 + c2 * 64, rc.P, rc.ke, rc.mw));
            mask32(sb, valid_bits(pos0 + c2 * 64 + 32, rc.P, rc.ke, rc.mw));
        }
        max32x2(sa, sb, mx);
    }
    const float mt = max16(mx) * rc.scale_log2;
    const bool need = mt > m_run + kRescaleThreshold;   // false if mt is -inf
    const float m_new = need ? mt : m_run;
    const float alpha = need ? ptx::ex2(m_run - m_new) : 1.f;   // 0 when m_run = -inf
    if (__any_sync(0xffffffffu, need) && !first) {
        if (!wait_o())
            return false;
        ptx::tc_fence_after();
        rescale_o(taddr_o, alpha);
    }
    l_run *= alpha;
    m_run = m_new;
    // P over the S columns already read: keys 64 c2 .. -> columns 32 c2 ..
    const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
    float lsum = 0.f;
#pragma unroll 1
    for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t sa[32], sb[32];
        ptx::tmem_ld32(taddr_s + c2 * 64, sa);
        ptx::tmem_ld32(taddr_s + c2 * 64 + 32, sb);
        ptx::tmem_wait_ld();
        if (masked) {
            mask32(sa, valid_bits(pos0 + c2 * 64, rc.P, rc.ke, rc.mw));
            mask32(sb, valid_bits(pos0 + c2 * 64 + 32, rc.P, rc.ke, rc.mw));
        }
        uint32_t pk[32];
        lsum += exp_pack64(sa, sb, rc.scale_log2, neg_m, pk);
        ptx::tmem_st32(taddr_s + c2 * 32, pk);
    }
    ptx::tmem_wait_st();
    l_run += lsum;
    return true;
}

// One key tile of the online softmax of the rows kernels, for this thread's
// query row: the BN scores in TMEM columns taddr_s are read into registers
// at once and masked where the tile reaches the tree or the range end.  P is
// written against the running max speculatively; the row max is only taken
// (and O rescaled) when some exponent may exceed the headroom -- the tile's
// sum above 2^64 or not finite, which always happens on a query tile's first
// key tile (m_run = -inf).  One exp loop, run a second time only by a warp
// that took the max.  `wait_prev` waits for the previous PV product before
// O is rescaled.  Returns false on abort.
template <int BN, typename WaitPrev>
__device__ __forceinline__ bool softmax_rows_tile(uint32_t taddr_s, uint32_t taddr_o, int pos0,
                                                  int P, int ke, const uint32_t (&mw)[4],
                                                  float scale_log2, bool first, float &m_run,
                                                  float &l_run, WaitPrev wait_prev)
{
    constexpr int NC = BN / 32;   // 32-column score chunks
    uint32_t sr[NC][32];
#pragma unroll
    for (int c = 0; c < NC; ++c)
        ptx::tmem_ld32(taddr_s + c * 32, sr[c]);
    ptx::tmem_wait_ld();
    if (!(pos0 + BN <= min(P, ke))) {   // only where the tree or the range end is
#pragma unroll
        for (int c = 0; c < NC; ++c)
            mask32(sr[c], valid_bits(pos0 + c * 32, P, ke, mw));
    }
    float lsum = 0.f;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
        lsum = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            uint32_t pk[16];
            lsum += exp_pack32(sr[c], scale_log2, neg_m, pk);
            ptx::tmem_st16(taddr_s + c * 16, pk);
        }
        const bool redo = !(lsum <= kLazyLimit) || m_run == -INFINITY;
        if (pass == 1 || !__any_sync(0xffffffffu, redo))
            break;
        float mx[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            mx[i] = -INFINITY;
#pragma unroll
        for (int c = 0; c < NC; c += 2)
            max32x2(sr[c], sr[c + 1], mx);
        const float mt = max16(mx) * scale_log2;
        const bool need = mt > m_run + kRescaleThreshold;   // false if mt is -inf
        const float m_new = need ? mt : m_run;
        const float alpha = need ? ptx::ex2(m_run - m_new) : 1.f;   // 0 when m_run = -inf
        if (__any_sync(0xffffffffu, need) && !first) {
            // O holds the products of the earlier key tiles: wait for the last.
            if (!wait_prev())
                return false;
            ptx::tc_fence_after();
            rescale_o(taddr_o, alpha);
        }
        l_run *= alpha;
        m_run = m_new;
        ptx::tmem_wait_st();   // the speculative P is overwritten next pass
    }
    l_run += lsum;
    ptx::tmem_wait_st();
    return true;
}

// Final O row (TMEM) -> output row (bf16, normalised) or split partial (fp32).
__device__ __forceinline__ void write_row(uint32_t taddr_o, float inv, bool row_ok, size_t row,
                                          int nsplit, int split, size_t nrows,
                                          __nv_bfloat16 *__restrict__ out,
                                          float *__restrict__ part_o, int col0, int ncols)
{
    for (int c = 0; c < ncols; c += 32) {
        uint32_t o[32];
        ptx::tmem_ld32(taddr_o + c, o);
        ptx::tmem_wait_ld();
        if (!row_ok)
            continue;
        if (nsplit == 1) {
            uint4 *dst = reinterpret_cast<uint4 *>(out + row * HD + col0 + c);
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
            float4 *dst = reinterpret_cast<float4 *>(part_o + ((size_t)split * nrows + row) * HD +
                                                     col0 + c);
#pragma unroll
            for (int v = 0; v < 8; ++v)
                dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv,
                                     __uint_as_float(o[4 * v + 1]) * inv,
                                     __uint_as_float(o[4 * v + 2]) * inv,
                                     __uint_as_float(o[4 * v + 3]) * inv);
        }
    }
}

// One 128-key tile of the online softmax split over two warps per TMEM lane
// quarter: this warp takes the 64 keys of its half (hf) of the tile, for the
// same 32 query rows as its partner warp, which takes the other half.  Both
// halves write P against the same running max m_run and keep their own part
// of the row sum (l_half).  Whether the row max must be taken (a half's P sum
// above 2^64 or not finite, always on the first tile) is decided for both at
// once: each warp publishes its ballot in the pair's exchange slots (by tile
// parity) and the two warps meet at a named barrier of 64 threads; when the
// max pass runs, each half publishes its rows' maxima the same way, so both
// take the same new maximum and rescale their 64 columns of O alike.
struct PairXchg {
    uint32_t vote[2][2];      // [exchange parity][half]: the warp's redo ballot
    float mx[2][2][32];       // [exchange parity][half][lane]: a value per row
};
static_assert(sizeof(PairXchg) == 528, "exchange slots");

// One exchange between the two warps of a lane quarter: each warp has
// written its slots of parity (n & 1) and arrives on the quarter's
// mbarrier; both wait for the phase (bounded, like every wait here).  The
// two warps make the same exchanges in the same order, so phase n of the
// barrier is exchange n; slots alternate by parity, so a warp writing the
// slots of exchange n + 2 has passed exchange n + 1, which its partner
// entered only after reading those of exchange n.
template <class Gm>
__device__ __forceinline__ bool pair_exchange(const Setup<Gm> &su, int quarter, int &n)
{
    warp_arrive(su.bars.pair(quarter));
    const bool ok = warp_wait(su.bars.pair(quarter), n & 1, su.abort_flag);
    ++n;
    return ok;
}

template <class Gm, typename WaitPrev>
__device__ __forceinline__ bool softmax_half_tile(const Setup<Gm> &su, uint32_t taddr_s,
                                                  uint32_t taddr_o, int pos0, int P, int ke,
                                                  const uint32_t (&mw)[4], float scale_log2,
                                                  bool first, int hf, int quarter, PairXchg *xc,
                                                  int &nx, float &m_run, float &l_half,
                                                  WaitPrev wait_prev)
{
    const int lane = threadIdx.x & 31;
    uint32_t sr[2][32];
    ptx::tmem_ld32(taddr_s, sr[0]);
    ptx::tmem_ld32(taddr_s + 32, sr[1]);
    ptx::tmem_wait_ld();
    if (!(pos0 + 64 <= min(P, ke))) {
        mask32(sr[0], valid_bits(pos0, P, ke, mw));
        mask32(sr[1], valid_bits(pos0 + 32, P, ke, mw));
    }
    float lsum = 0.f;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
        lsum = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t pk[16];
            lsum += exp_pack32(sr[c], scale_log2, neg_m, pk);
            ptx::tmem_st16(taddr_s + c * 16, pk);
        }
        if (pass == 1)
            break;
        const bool redo = !(lsum <= kLazyLimit) || m_run == -INFINITY;
        const uint32_t vote = __ballot_sync(0xffffffffu, redo);
        int par = nx & 1;
        if (lane == 0)
            xc->vote[par][hf] = vote;
        if (!pair_exchange(su, quarter, nx))
            return false;
        if ((xc->vote[par][0] | xc->vote[par][1]) == 0u)
            break;
        float mx[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            mx[i] = -INFINITY;
        max32x2(sr[0], sr[1], mx);
        par = nx & 1;
        xc->mx[par][hf][lane] = max16(mx);
        if (!pair_exchange(su, quarter, nx))
            return false;
        const float mt = fmaxf(xc->mx[par][0][lane], xc->mx[par][1][lane]) * scale_log2;
        const bool need = mt > m_run + kRescaleThreshold;   // false if mt is -inf
        const float m_new = need ? mt : m_run;
        const float alpha = need ? ptx::ex2(m_run - m_new) : 1.f;   // 0 when m_run = -inf
        if (__any_sync(0xffffffffu, need) && !first) {
            // O holds the products of the earlier key tiles: wait for the last,
            // then rescale this half's 64 columns of it.
            if (!wait_prev())
                return false;
            ptx::tc_fence_after();
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(taddr_o + c * 32, o);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k)
                    o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                ptx::tmem_st32(taddr_o + c * 32, o);
            }
        }
        l_half *= alpha;
        m_run = m_new;
        ptx::tmem_wait_st();   // the speculative P is overwritten next pass
    }
    l_half += lsum;
    ptx::tmem_wait_st();
    return true;
}

// ============================================================ rows kernel
// More than 128 packed rows: one 128-row query tile per CTA; warp 0 the TMA
// producer, warp 1 the MMA issuer, then the softmax warps.  NS score buffers
// of BN columns each, then O: the MMA warp keeps the scores of the next NS - 1
// key tiles ready while the softmax works on tile j.  Instances:
//   * 128-key tiles, NS = 3, one CTA per SM:
//         TMEM S0 [0,128) | S1 [128,256) | S2 [256,384) | O [384,512)
//     with SW = 1 softmax warp per TMEM lane quarter (each thread a whole
//     row of 128 scores), or SW = 2 (8 softmax warps, two per SM
//     sub-partition: each takes one 64-key half of the tile for 32 rows, so
//     a sub-partition interleaves two warps' exponentials; P of each half is
//     written over that half's own score columns);
//   * 64-key tiles, NS = 2, two CTAs per SM (each with 256 TMEM columns and
//     97 KB of shared memory): S0 [0,64) | S1 [64,128) | O [128,256).  The
//     two CTAs' MMA warps feed one tensor pipe and their softmax warps share
//     the sub-partitions, so one CTA's barrier waits and exp latency are
//     covered by the other's work.
// MMA order: QK_0 .. QK_{NS-1}, then per tile j: PV_j QK_{j+NS}; P_j is read
// out of S_{j%NS} by PV_j before QK_{j+NS}, issued after it by the same
// thread, overwrites it.  QK_i commits to s_full[i%NS], PV_j to o_ready[j%NS]
// (the producer reuses ring slots on those same barriers).  The softmax at
// tile j waits for "PV_{j-1} done" on o_ready[(j-1)%NS]: the phase before it
// there is PV_{j-1-NS}, issued before QK_j, whose completion the softmax has
// already seen, and the phase after it needs P_{j-1+NS}, not yet written --
// so the wait names a phase that can be neither stale nor ahead.
template <int SW>
constexpr int rows_threads() { return 64 + 128 * SW; }

template <class Gm, int NS, int kMinBlocks, int SW>
__global__ void __launch_bounds__(rows_threads<SW>(), kMinBlocks)
    tree_attn_rows_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __nv_bfloat16 *__restrict__ q,
                          const int32_t *__restrict__ prefix_len,
                          const int32_t *__restrict__ n_nodes, const uint32_t *__restrict__ mask,
                          int Tmax, int Hq, int Hkv, int Lmax, int W, float scale_log2,
                          int keys_per_split, int nsplit, __nv_bfloat16 *__restrict__ out,
                          float *__restrict__ part_o, float2 *__restrict__ part_ml,
                          int32_t *dev_status, KvPages pages)
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
    if (rb * BQ >= R || kb >= ke)
        return;   // no rows or no keys: the partials stay empty
    constexpr int BN = Gm::BN, NSK = Gm::NSK, NSV = Gm::NSV;
    static_assert(NS * BN + HD <= (int)Gm::kTmemCols && BN % 64 == 0, "TMEM layout");
    static_assert(SW == 1 || (SW == 2 && BN == 128), "split softmax: 128-key tiles");
    static_assert(NS == NSK, "the producer reuses K slots on the score barriers");
    const int ntiles = (ke - kb + BN - 1) / BN;
    // arrivals: every softmax warp loads its part of Q and publishes its P
    const Setup<Gm> su = cta_setup<Gm>(smem_raw, 4 * SW, 4 * SW);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto col_s = [](int i) { return (uint32_t)(i % NS) * (uint32_t)BN; };
    constexpr uint32_t kO = NS * BN;

    if (warp == 0) {
        const PageCache pc = stage_pages(su, pages, b, kb, min(ke, P + T), lane);
        if (lane == 0)
            produce_kv<Gm, NS>(su, &tmK, &tmV, b, hk, Hkv, kb, ntiles, pages, pc, P + T,
                               dev_status);
    } else if (warp == 1) {
        // Every cycle the MMA-issuing thread spends between MMAs leaves the
        // tensor pipe idle (it queues little ahead of the thread), and a
        // wait costs a barrier round trip even when the phase is complete.
        // So the barriers of V_{j+1} and K_{j+NS}, which have usually landed
        // long before, are tested while the MMAs before them are issued, and
        // only P_j (the softmax's, the one that is often late) is waited for
        // in line.  The whole warp polls (a lane-0 poll with the other lanes
        // held at a shuffle measured slower).
        auto kbar = [&](int i) { return su.bars.k_full(i % NSK); };
        auto kpar = [&](int i) { return (uint32_t)(i / NSK) & 1u; };
        auto vbar = [&](int i) { return su.bars.v_full(i % NSV); };
        auto vpar = [&](int i) { return (uint32_t)(i / NSV) & 1u; };
        bool ok = warp_wait(su.bars.q_full(), 0, su.abort_flag);
        ptx::tc_fence_after();
        // QK_i commits to s_full[i % NS], PV_j to o_ready[j % NS]
        for (int i = 0; ok && i < min(NS, ntiles); ++i) {
            ok = warp_wait(kbar(i), kpar(i), su.abort_flag);
            ptx::tc_fence_after();
            if (ok)
                issue_qk<Gm, false>(su, lane, col_s(i), i, su.bars.s_full(i % NS));
        }
        // tests of phases whose previous phase this warp has already waited
        // for (V_{j+1-NSV} before PV_{j+1-NSV}, K_j before QK_j), and whose
        // next phase needs a product not yet issued (PV_{j+1}, QK_{j+NS})
        uint32_t v_tested = ntiles > 0 ? ptx::mbar_test(vbar(0), vpar(0)) : 1u;
        for (int j = 0; ok && j < ntiles; ++j) {
            if (!warp_wait(su.bars.p_full(j % NS), (j / NS) & 1, su.abort_flag) ||
                !warp_wait_tested(v_tested, vbar(j), vpar(j), su.abort_flag)) {
                ok = false;
                break;
            }
            const int i = j + NS;
            const uint32_t k_tested = i < ntiles ? ptx::mbar_test(kbar(i), kpar(i)) : 1u;
            issue_pv<Gm, false, SW == 2>(su, lane, col_s(j), kO, j, j > 0,
                                         P + T - (kb + j * BN), su.bars.o_ready(j % NS));
            if (i < ntiles && !warp_wait_tested(k_tested, kbar(i), kpar(i), su.abort_flag)) {
                ok = false;
                break;
            }
            v_tested = j + 1 < ntiles ? ptx::mbar_test(vbar(j + 1), vpar(j + 1)) : 1u;
            if (i < ntiles) {
                ptx::tc_fence_after();
                issue_qk<Gm, false>(su, lane, col_s(i), i, su.bars.s_full(i % NS));
            }
        }
    } else {
        // softmax warps: one query row per thread == TMEM lane; with SW = 2
        // the two warps of a lane quarter split the tile's keys (hf = half)
        const int quarter = warp & 3;
        const int hf = SW == 2 ? (warp - 2) >> 2 : 0;
        const int t = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int r = rb * BQ + t;
        // the row's q / out / mask entries (bounds of the checked build:
        // every one of them is in range iff the q row index is)
        const bool row_ok = r < R && in_bounds(((long long)b * Tmax + r / G) * Hq + hk * G + r % G,
                                               (long long)gridDim.y / Hkv * Tmax * Hq, dev_status);
        const int u = row_ok ? r / G : 0;
        const int h = hk * G + (row_ok ? r % G : 0);
        load_q_row<Gm, SW>(su, q, row_ok, (((size_t)b * Tmax + u) * Hq + h) * HD, t, hf);
        warp_arrive(su.bars.q_full());
        uint32_t mw[4];
#pragma unroll
        for (int w = 0; w < 4; ++w)
            mw[w] = (row_ok && w < W) ? mask[((size_t)b * Tmax + u) * W + w] : 0u;
        const uint32_t taddr_o = su.tmem + lane_off + kO + hf * 64;
        PairXchg *xc = reinterpret_cast<PairXchg *>(su.gbase + Gm::kOffXchg) + quarter;
        // PV_i done (o_ready[i % NS] completes once per tile of that class)
        auto wait_pv = [&](int i) {
            return warp_wait(su.bars.o_ready(i % NS), (i / NS) & 1, su.abort_flag);
        };
        float m_run = -INFINITY, l_run = 0.f;
        int nx = 0;   // pair exchanges made
        bool ok = true;
        // S_{j+1} is tested at the start of tile j and read after it: QK_{j+1}
        // completes long before (it was issued after PV_{j+1-NS}), so the wait
        // costs a vote; the phase before it (QK_{j+1-NS}) was waited for at
        // tile j+1-NS, and the one after it needs this warp's P_{j+1}.
        uint32_t s_tested = ntiles > 0 ? ptx::mbar_test(su.bars.s_full(0), 0) : 1u;
        for (int j = 0; ok && j < ntiles; ++j) {
            if (!warp_wait_tested(s_tested, su.bars.s_full(j % NS), (j / NS) & 1,
                                  su.abort_flag)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            s_tested = j + 1 < ntiles
                           ? ptx::mbar_test(su.bars.s_full((j + 1) % NS), ((j + 1) / NS) & 1)
                           : 1u;
            auto wait_prev = [&]() { return wait_pv(j - 1); };
            if (SW == 1)
                ok = softmax_rows_tile<BN>(su.tmem + lane_off + col_s(j), taddr_o, kb + j * BN,
                                           P, ke, mw, scale_log2, j == 0, m_run, l_run,
                                           wait_prev);
            else
                ok = softmax_half_tile<Gm>(su, su.tmem + lane_off + col_s(j) + hf * 64, taddr_o,
                                       kb + j * BN + hf * 64, P, ke, mw, scale_log2, j == 0, hf,
                                       quarter, xc, nx, m_run, l_run, wait_prev);
            if (!ok)
                break;
            ptx::tc_fence_before();
            warp_arrive(su.bars.p_full(j % NS));
        }
        bool done = ok && wait_pv(ntiles - 1);
        if (SW == 2 && done) {
            // the row sum is the two halves' sums (a warp that gave up skips
            // this; its partner's bounded wait then sees the abort flag)
            const int par = nx & 1;
            xc->mx[par][hf][lane] = l_run;
            done = pair_exchange(su, quarter, nx);
            l_run = xc->mx[par][0][lane] + xc->mx[par][1][lane];
        }
        if (done) {
            ptx::tc_fence_after();
            const size_t row = ((size_t)b * Tmax + u) * Hq + h;
            const size_t nrows = (size_t)gridDim.y / Hkv * Tmax * Hq;
            const float inv = nsplit == 1 ? (l_run > 0.f ? 1.f / l_run : 0.f) : 1.f;
            write_row(taddr_o, inv, row_ok, row, nsplit, split, nrows, out, part_o, hf * 64,
                      HD / SW);
            if (row_ok && nsplit > 1 && hf == 0)
                part_ml[(size_t)split * nrows + row] = make_float2(m_run, l_run);
        }
    }
    cta_teardown(su, dev_status);
}

// ======================================================== key-split kernel
// At most 128 packed rows: softmax group s (warps 4+4s .. 7+4s) takes the key
// tiles s, s+2, s+4, ... of the CTA's range with its own S_s and O_s.
// TMEM: S0 [0,128) | S1 [128,256) | O0 [256,384) | O1 [384,512).
// MMA order: QK(0) QK(1) | PV(0) QK(2) | PV(1) QK(3) | ...  (tile k belongs to
// group k & 1; S_s is reused after PV of its previous tile, in issue order).
__global__ void __launch_bounds__(kSplitThreads, 1)
    tree_attn_keysplit_kernel(const __grid_constant__ CUtensorMap tmK,
                              const __grid_constant__ CUtensorMap tmV,
                              const __nv_bfloat16 *__restrict__ q,
                              const int32_t *__restrict__ prefix_len,
                              const int32_t *__restrict__ n_nodes,
                              const uint32_t *__restrict__ mask, int Tmax, int Hq, int Hkv,
                              int Lmax, int W, float scale_log2, int keys_per_split, int nsplit,
                              __nv_bfloat16 *__restrict__ out, float *__restrict__ part_o,
                              float2 *__restrict__ part_ml, int32_t *dev_status,
                              KvPages pages)
{
    extern __shared__ uint8_t smem_raw[];
    const int pair = blockIdx.y, split = blockIdx.z;
    const int b = pair / Hkv, hk = pair % Hkv;
    const int G = Hq / Hkv;
    const int T = n_nodes[b], P = prefix_len[b];
    if (!tree_header_ok(T, Tmax) || P < 0 || P + T > Lmax) {
        if (split == 0 && hk == 0 && threadIdx.x == 0)
            flag(dev_status, TSD_DEV_BAD_PREFIX);
        return;
    }
    const int R = T * G;
    const int kb = split * keys_per_split;
    const int ke = min(kb + keys_per_split, P + T);
    if (R <= 0 || kb >= ke)
        return;
    using Gm = Wide;
    constexpr int BN = Gm::BN, NSK = Gm::NSK, NSV = Gm::NSV;
    const int ntiles = (ke - kb + BN - 1) / BN;
    const Setup<Gm> su = cta_setup<Gm>(smem_raw, 8, 4);   // arrivals: softmax warps
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto col_s = [](int s) { return (uint32_t)s * 128u; };
    auto col_o = [](int s) { return 256u + (uint32_t)s * 128u; };

    if (warp == 0) {
        const PageCache pc = stage_pages(su, pages, b, kb, min(ke, P + T), lane);
        if (lane == 0)
            produce_kv<Gm, 0>(su, &tmK, &tmV, b, hk, Hkv, kb, ntiles, pages, pc, P + T,
                              dev_status);
    } else if (warp == 1) {
        bool ok = warp_wait(su.bars.q_full(), 0, su.abort_flag);
        ptx::tc_fence_after();
        auto qk = [&](int k) -> bool {
            if (!warp_wait(su.bars.k_full(k % NSK), (k / NSK) & 1, su.abort_flag))
                return false;
            ptx::tc_fence_after();
            issue_qk(su, lane, col_s(k & 1), k, su.bars.s_full(k & 1));
            return true;
        };
        if (ok)
            ok = qk(0);
        if (ok && ntiles > 1)
            ok = qk(1);
        for (int k = 0; ok && k < ntiles; ++k) {
            const int s = k & 1;
            if (!warp_wait(su.bars.p_full(s), (k >> 1) & 1, su.abort_flag) ||
                !warp_wait(su.bars.v_full(k % NSV), (k / NSV) & 1, su.abort_flag)) {
                ok = false;
                break;
            }
            issue_pv(su, lane, col_s(s), col_o(s), k, k >= 2, P + T - (kb + k * BN),
                     su.bars.o_ready(s));
            if (k + 2 < ntiles)
                ok = qk(k + 2);
        }
    } else if (warp >= 4) {
        const int s = (warp - 4) >> 2;   // group
        const int quarter = warp & 3;
        const int t = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const bool row_ok = t < R && in_bounds(((long long)b * Tmax + t / G) * Hq + hk * G + t % G,
                                               (long long)gridDim.y / Hkv * Tmax * Hq, dev_status);
        const int u = row_ok ? t / G : 0;
        const int h = hk * G + (row_ok ? t % G : 0);
        if (s == 0)
            load_q_row(su, q, row_ok, (((size_t)b * Tmax + u) * Hq + h) * HD, t);
        warp_arrive(su.bars.q_full());
        RowCtx rc;
        rc.P = P;
        rc.ke = ke;
        rc.scale_log2 = scale_log2;
#pragma unroll
        for (int w = 0; w < 4; ++w)
            rc.mw[w] = (row_ok && w < W) ? mask[((size_t)b * Tmax + u) * W + w] : 0u;
        const int my_tiles = (ntiles - s + 1) / 2;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int mi = 0; ok && mi < my_tiles; ++mi) {
            if (!warp_wait(su.bars.s_full(s), mi & 1, su.abort_flag)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            auto wait_o = [&]() { return warp_wait(su.bars.o_ready(s), (mi - 1) & 1, su.abort_flag); };
            ok = softmax_tile(su.tmem + lane_off + col_s(s), su.tmem + lane_off + col_o(s),
                              kb + (2 * mi + s) * BN, rc, mi == 0, m_run, l_run, wait_o);
            if (!ok)
                break;
            ptx::tc_fence_before();
            warp_arrive(su.bars.p_full(s));
        }
        const bool have = ok && my_tiles > 0 &&
                          warp_wait(su.bars.o_ready(s), (my_tiles - 1) & 1, su.abort_flag);
        ptx::tc_fence_after();
        // Merge (m, l) of the two groups through shared memory in the Q tile.
        // Q is only free once group 0 has seen its last product: every QK
        // (the only reader of Q) is issued before that PV, while group 1 may
        // have had no tile at all and get here at once.
        ptx::named_barrier(1, 2 * BQ);
        float2 *ml = reinterpret_cast<float2 *>(su.gbase + kOffQ);
        ml[s * BQ + t] = make_float2(have ? m_run : -INFINITY, have ? l_run : 0.f);
        ptx::named_barrier(1, 2 * BQ);
        const float2 a = ml[t], c2 = ml[BQ + t];
        const float M = fmaxf(a.x, c2.x);
        const float w0 = a.y > 0.f ? ptx::ex2(a.x - M) : 0.f;
        const float w1 = c2.y > 0.f ? ptx::ex2(c2.x - M) : 0.f;
        const float L = a.y * w0 + c2.y * w1;
        const float inv = nsplit == 1 ? (L > 0.f ? 1.f / L : 0.f) : 1.f;
        const size_t row = ((size_t)b * Tmax + u) * Hq + h;
        const size_t nrows = (size_t)gridDim.y / Hkv * Tmax * Hq;
        // group s writes head_dim columns [64 s, 64 s + 64)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint32_t col = s * 64 + c * 32;
            uint32_t o0[32], o1[32];
            ptx::tmem_ld32(su.tmem + lane_off + col_o(0) + col, o0);
            ptx::tmem_ld32(su.tmem + lane_off + col_o(1) + col, o1);
            ptx::tmem_wait_ld();
            if (!row_ok)
                continue;
            float o[32];
#pragma unroll
            for (int k = 0; k < 32; ++k)
                o[k] = ((w0 > 0.f ? __uint_as_float(o0[k]) * w0 : 0.f) +
                        (w1 > 0.f ? __uint_as_float(o1[k]) * w1 : 0.f)) * inv;
            if (nsplit == 1) {
                uint4 *dst = reinterpret_cast<uint4 *>(out + row * HD + col);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    uint4 x;
                    x.x = ptx::pack_bf16(o[8 * v + 0], o[8 * v + 1]);
                    x.y = ptx::pack_bf16(o[8 * v + 2], o[8 * v + 3]);
                    x.z = ptx::pack_bf16(o[8 * v + 4], o[8 * v + 5]);
                    x.w = ptx::pack_bf16(o[8 * v + 6], o[8 * v + 7]);
                    dst[v] = x;
                }
            } else {
                float4 *dst = reinterpret_cast<float4 *>(
                    part_o + ((size_t)split * nrows + row) * HD + col);
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    dst[v] = make_float4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
            }
        }
        if (row_ok && nsplit > 1 && s == 0)
            part_ml[(size_t)split * nrows + row] = make_float2(M, L);
    }
    cta_teardown(su, dev_status);
}

// ------------------------------------------------------------------ host
struct UmmaPlan {
    bool keysplit;   // at most 128 packed rows
    bool paired;     // rows kernel with 64-key tiles, two CTAs per SM
    int sw;          // 128-key rows kernel: softmax warps per TMEM lane quarter
    int nrb, nsplit, keys_per_split;
};

// Softmax warps per TMEM lane quarter of the 128-key rows kernel: 1, or 2
// when the environment variable TSD_ATTN_SOFTMAX_WARPS is "2" (read at every
// launch).
int rows_softmax_warps()
{
    const char *e = std::getenv("TSD_ATTN_SOFTMAX_WARPS");
    return (e && e[0] == '2' && e[1] == '\0') ? 2 : 1;
}


// Rows-kernel instance for more than 128 packed rows: 1 = 128-key tiles at
// one CTA per SM (default), 2 = 64-key tiles at two CTAs per SM when the
// environment variable TSD_ATTN_ROWS_VARIANT is "2" (read at every launch,
// so that one process can run and compare both).
int rows_variant()
{
    const char *e = std::getenv("TSD_ATTN_ROWS_VARIANT");
    return (e && e[0] == '2' && e[1] == '\0') ? 2 : 1;
}

// At most 128 packed rows: the paired 64-key rows kernel (default), or the
// key-split kernel when TSD_ATTN_SMALL_VARIANT is "keysplit".
bool small_paired()
{
    const char *e = std::getenv("TSD_ATTN_SMALL_VARIANT");
    return !(e && std::strcmp(e, "keysplit") == 0);
}

// Kernel choice and grid.  More than 128 packed rows go to the rows kernel:
// 64-key tiles at two CTAs per SM, or 128-key tiles at one.  Splits of the
// key range balance the grid over the CTA slots.
UmmaPlan umma_plan(const AttnArgs &a, int num_sms)
{
    UmmaPlan p;
    const int G = a.Hq / a.Hkv;
    const bool small = a.Tmax * G <= BQ;
    p.keysplit = small && !small_paired();
    p.paired = small ? !p.keysplit : rows_variant() == 2;
    p.sw = (p.keysplit || p.paired) ? 1 : rows_softmax_warps();
    p.nrb = p.keysplit ? 1 : (a.Tmax * G + BQ - 1) / BQ;
    const int bn = p.paired ? Half::BN : Wide::BN;
    const int slots = num_sms * (p.paired ? 2 : 1);
    const long base = (long)p.nrb * a.B * a.Hkv;
    const int tiles = (a.Lmax + bn - 1) / bn;
    // Cost of ns splits in tile times.  One CTA per SM: waves x (tiles per
    // CTA + fixed cost).  Two per SM: the scheduler refills a slot as soon as
    // a CTA ends and a CTA alone on an SM runs faster, so the wave count is
    // taken fractionally (but at least one CTA length), and a split pays for
    // its fp32 partials and the combine pass.
    const int fixed = 256 / bn;
    int best = 1;
    double best_cost = 1e30;
    for (int ns = 1; ns <= 64 && ns <= tiles; ++ns) {
        const long units = base * ns;
        const int per = (tiles + ns - 1) / ns;
        double cost;
        if (p.paired)
            cost = std::max((double)units / slots, 1.0) * (per + fixed) + (ns > 1 ? fixed : 0);
        else
            cost = (double)((units + slots - 1) / slots) * (per + fixed);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = ns;
        }
    }
    // TSD_ATTN_SPLITS=n forces n key-range splits (1..64, at most one per
    // tile) in place of the cost model's choice.
    if (const char *e = std::getenv("TSD_ATTN_SPLITS")) {
        const int n = std::atoi(e);
        if (n >= 1)
            best = std::min(std::min(n, 64), tiles);
    }
    p.nsplit = best;
    p.keys_per_split = ((tiles + best - 1) / best) * bn;
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
// [planes][rows][128] bf16 viewed as a 3-D tensor, boxes of [1][box_rows][64]:
// a contiguous cache has planes = B * Hkv and rows = Lmax, a paged pool has
// planes = num_pages * Hkv and rows = page_size.
bool make_kv_map(CUtensorMap *m, const void *ptr, int rows, int planes, int box_rows)
{
    auto fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)rows, (cuuint64_t)planes};
    cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)rows * HD * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The kernels' shared-memory limits are attributes of the current device's
// copy of each kernel: raised once per device (a process may drive several).
cudaError_t set_smem_attributes()
{
    constexpr int kMaxDevices = 64;
    static std::atomic<bool> done[kMaxDevices];
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    if (done[dev].load())
        return cudaSuccess;
    const void *wide_kernels[] = {(const void *)tree_attn_rows_kernel<Wide, 3, 1, 1>,
                                  (const void *)tree_attn_rows_kernel<Wide, 3, 1, 2>,
                                  (const void *)tree_attn_keysplit_kernel};
    for (const void *k : wide_kernels)
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Wide::kSmemBytes);
    const void *half_kernels[] = {(const void *)tree_attn_rows_kernel<Half, 2, 2, 1>};
    for (const void *k : half_kernels) {
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Half::kSmemBytes);
        // two CTAs per SM need the largest shared-memory carve-out
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       (int)cudaSharedmemCarveoutMaxShared);
    }
    if (err == cudaSuccess)
        done[dev].store(true);
    return err;
}

}  // namespace

bool umma_attention_supported(const AttnArgs &a)
{
    // bf16, head_dim 128, and a packed query block large enough to feed the
    // tensor cores (smaller blocks stay on the CUDA-core path).
    return a.dtype == TSD_BF16 && a.D == HD && a.Tmax * (a.Hq / a.Hkv) >= 8;
}

void umma_attention_plan(const AttnArgs &a, int num_sms, int32_t out[4])
{
    const UmmaPlan p = umma_plan(a, num_sms);
    out[0] = p.keysplit ? TSD_PLAN_KEYSPLIT
                        : (p.paired ? TSD_PLAN_ROWS64
                                    : (p.sw == 2 ? TSD_PLAN_ROWS128_PAIRED : TSD_PLAN_ROWS128));
    out[1] = p.nrb;
    out[2] = p.nsplit;
    out[3] = p.keys_per_split;
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
    const bool paged = a.pages.table != nullptr;
    const int rows = paged ? a.pages.page_size : a.Lmax;
    const int planes = paged ? a.pages.num_pages * a.Hkv : a.B * a.Hkv;
    const int bn = p.paired ? Half::BN : Wide::BN;
    const int box_rows = paged ? std::min(bn, a.pages.page_size) : bn;
    if (!make_kv_map(&tmK, a.k, rows, planes, box_rows) ||
        !make_kv_map(&tmV, a.v, rows, planes, box_rows))
        return TSD_ERR_CUDA;
    TSD_CUDA_TRY(set_smem_attributes());
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
    const float sl2 = a.scale * kLog2e;
    const int W = (a.Tmax + 31) / 32;
    if (p.keysplit)
        tree_attn_keysplit_kernel<<<grid, kSplitThreads, Wide::kSmemBytes, stream>>>(
            tmK, tmV, static_cast<const __nv_bfloat16 *>(a.q), a.prefix_len, a.n_nodes, a.mask,
            a.Tmax, a.Hq, a.Hkv, a.Lmax, W, sl2, p.keys_per_split, p.nsplit,
            static_cast<__nv_bfloat16 *>(a.out), part_o, part_ml, a.dev_status, a.pages);
    else {
        auto kern = p.paired    ? tree_attn_rows_kernel<Half, 2, 2, 1>
                    : p.sw == 2 ? tree_attn_rows_kernel<Wide, 3, 1, 2>
                                : tree_attn_rows_kernel<Wide, 3, 1, 1>;
        const int threads = p.sw == 2 ? rows_threads<2>() : rows_threads<1>();
        const uint32_t smem = p.paired ? Half::kSmemBytes : Wide::kSmemBytes;
        kern<<<grid, threads, smem, stream>>>(
            tmK, tmV, static_cast<const __nv_bfloat16 *>(a.q), a.prefix_len, a.n_nodes, a.mask,
            a.Tmax, a.Hq, a.Hkv, a.Lmax, W, sl2, p.keys_per_split, p.nsplit,
            static_cast<__nv_bfloat16 *>(a.out), part_o, part_ml, a.dev_status, a.pages);
    }
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
