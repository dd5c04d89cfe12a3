// attn_tc_bwd.cu -- a6 routed attention backward on the tcgen05 tensor cores
// (bf16 inputs, d = 64 or 128, float32 accumulation).
//
// Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com),
// section "What HGA does differently": the router has no learned weights, so
// the gradients reach Q, K and V exactly as in dense attention over the routed
// key set; the segment-wise backward of the same section detaches older KV,
// so key gradients are kept for the segment's own tokens only.  The routing
// of the forward is reused unchanged.
//
// One CTA owns one (batch, kv-head, query block) and a pair of q-heads: one
// M-tile of 128 query rows.  For each 64-key tile (8 routed groups, or the
// own chunk with the causal mask):
//     S   = Q K^T, dP = dO V^T        tcgen05.mma -> tensor memory
//     P   = exp2(S*c - lse), dS = P (dP - D)   row per thread; dS goes back
//           over S in tensor memory as bf16 hi + lo parts (~14-bit operand)
//     dQ += dS K                      A = dS (tensor memory), B = K (MN-major)
// and for the tiles holding segment keys, with P and dS also written to
// shared memory (hi + lo):
//     dV^T = dO^T P, dK^T = Q^T dS    A = dO / Q read MN-major, B = P / dS
// dV^T and dK^T (d on the tensor-memory lanes, keys on the columns) are added
// to the float32 dV_seg / dK_seg rows of the segment's keys with coalesced
// atomics; tiles of detached history skip both products.
//
// Tile order: an item runs its tiles from the own chunk down to the first
// routed tile, so the tiles holding segment keys (the own chunk and the last
// routed tiles, groups being ascending) come first.  Once their products are
// done the item's P/dS buffer is free and the next item's Q and dO load into
// it: two 64 KB buffers swap the Q/dO and P/dS roles from item to item, and
// the next item's S/dP products start while this item's history tiles run.
//
// Warp roles (608 threads): warps 0-15 compute P and dS (row 32*(w%4)+lane,
// 16-key quarter w/4), add a segment tile's dK/dV while the next tile's MMAs
// run and write dQ at the end of an item; warp 16 loads Q / dO and the K/V
// tiles (TMA gathers of 8-row groups); warp 17 owns tensor memory and issues
// the gradient MMAs (dQ, dV^T, dK^T); warp 18 issues S / dP.  A single
// issuing thread serialised the two streams: each tcgen05.mma takes it
// 70-90 cycles to issue, and its waits (the compute warps' hand-off, the
// next tile's K / V) delayed everything queued behind them.  With two
// issuers, S / dP of tile t + 2 go out as soon as its operands have landed
// and dQ of tile t, which reads dS from the same tensor-memory buffer, has
// completed (an mbarrier the gradient issuer commits).  Tensor memory (512 columns): S and dP
// double-buffered (4 x 64), dQ (128), dV^T (64), dK^T (64).  K and V load
// into separate rings: four K stages (K is read by S, two tiles ahead, and
// by dQ) and two V stages (V is read by dP only and released as S / dP
// complete), so each load is issued about two tiles before its use; with
// the two Q/dO <-> P/dS buffers they fill 224 KB of shared memory.
#include <algorithm>

#include "check.cuh"
#include "hga_internal.cuh"
#include "sm100.cuh"
#include "window_union.cuh"

namespace hga {
namespace {

using namespace sm100;

// The kernel's layout is 128 columns wide.  With d = 64 the second 64-column
// half of every Q / dO / K / V box lies past the tensor maps' width and the
// TMA fills it with zeros, so S, dP and the products stay exact; dQ and the
// dK / dV rows are written for the first d columns only.
constexpr int D = 128;
constexpr int H = 2;                  // 64-column halves of d
constexpr int kKStages = 4;            // K is read by S (issued two tiles ahead) and dQ
constexpr int kVStages = 2;            // V only by dP: released as S / dP complete
constexpr int kKeys = 64;
constexpr int kComputeWarps = 16;     // 4 per lane quadrant, one 16-key quarter each
constexpr int kCompute = 32 * kComputeWarps;
constexpr int kProducerWarp = kComputeWarps, kMmaWarp = kComputeWarps + 1, kSdpWarp = kComputeWarps + 2;
constexpr int kThreads = 32 * (kComputeWarps + 3);
constexpr float kLog2e = 1.4426950408889634f;

enum : int {
    kSiteQ = 201, kSiteFull, kSiteEmpty, kSiteSdp, kSitePs, kSiteKv, kSiteDrained, kSiteFinal, kSiteDrain,
    kSiteQfree, kSiteDqfree, kSitePfree, kSiteDqs, kSiteSfree, kSiteFinalSdp, kSiteDsum
};

template <int KST>                   // K stages
struct BwdSmem {
    static constexpr int kRows128 = 128 * 128;        // 128 rows x 128 B
    static constexpr int kKVHalf = kKeys * 128;       // 64 keys x 128 B
    // Two buffers of 64 KB.  As Q/dO: Q [2 halves][128 rows][64], then dO
    // alike.  As P/dS: P hi, P lo, dS hi, dS lo, each [128 rows][64 keys].
    static constexpr int kX = 4 * kRows128;
    static constexpr int x_off = 0;
    static constexpr int k_off = x_off + 2 * kX;
    static constexpr int v_off = k_off + KST * H * kKVHalf;
    static constexpr int bar_off = v_off + kVStages * H * kKVHalf;
    static constexpr int n_bars = 30;
    static constexpr int tab_off = (bar_off + 8 * n_bars + 15) & ~15;   // int4 (item, n_g, n_seg) of the CTA's first items
    static constexpr int tmem_slot_off = tab_off + 16 * 64;
    static constexpr int bytes = tmem_slot_off + 16;
    static constexpr int alloc = bytes + 1024;
    // Strictly causal variant: the window's union of routed groups
    // (wu::bytes, sized at launch).
    static constexpr int union_off = (bytes + 15) & ~15;
};
static_assert(BwdSmem<kKStages>::alloc <= 227 * 1024, "shared memory");
static_assert(BwdSmem<kKStages>::tab_off % 16 == 0 && BwdSmem<kKStages>::bar_off % 8 == 0,
              "int4 table and mbarrier alignment");
static_assert(BwdSmem<3>::union_off % 16 == 0, "union alignment");

// mbarriers: q[2], kfull / kempty[kKStages], vfull / vempty[kVStages], sdp[2],
// ps[2], kv, drained, pfree, qfree, dqfree, final, dqs_full, dqs_free, sfree[2],
// final_sdp, dsum (causal: the rows' partial sums D are in).
constexpr int kBarQ = 0, kBarKFull = 2, kBarKEmpty = kBarKFull + kKStages, kBarVFull = kBarKEmpty + kKStages,
              kBarVEmpty = kBarVFull + kVStages, kBarSdp = kBarVEmpty + kVStages, kBarPs = kBarSdp + 2,
              kBarKv = kBarPs + 2, kBarDrained = kBarKv + 1, kBarPfree = kBarKv + 2, kBarQfree = kBarKv + 3,
              kBarDqfree = kBarKv + 4, kBarFinal = kBarKv + 5, kBarDqsFull = kBarKv + 6,
              kBarDqsFree = kBarKv + 7, kBarSfree = kBarKv + 8, kBarFinalSdp = kBarSfree + 2,
              kBarDsum = kBarFinalSdp + 1;
static_assert(kBarDsum + 1 == BwdSmem<kKStages>::n_bars, "barrier count");

// Tensor-memory columns.
constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256, kColDV = 384, kColDK = 448;

struct BwdArgs {
    const int32_t* gidx;
    const int32_t* sched;      // CTA c's k-th item at sched[k * gridDim.x + c] (causal: may be null, item c)
    const float* lse;
    const float* Drow;         // block path: the row sums D of the row-dot launch
    float* dQ;
    float* dK;
    float* dV;
    int Hq, Hkv, G, wg, d;     // d: head dim of the tensors (64 or 128)
    int64_t T_hist, T_seg, nQB, n_items;
    int64_t cap;               // K / V rows per (batch, kv-head)
    int64_t nWin, n_groups;    // strictly causal variant: windows per (b, g); groups of the context
    const float* O;            // strictly causal variant: O, for the row sums D = rowsum(dO * O)
    const __nv_bfloat16* dO;
    int q_rows;
    float scale, scale_log2;
};

// One work item: a (batch, kv-head, query block) and a pair of its q-heads.
// Processing index p visits key tile t = nt - 1 - p; tiles p < n_seg hold
// segment keys.
struct Item {
    int u, bg, qb, head0, n_g, n_seg;   // u = bg * nQB + qb, bg = b * Hkv + g
    int w0, own0;                       // first query (in the segment) of the rows; first token of the own chunk
    __device__ __forceinline__ int n_rt() const { return (n_g + 7) / 8; }
    __device__ __forceinline__ int nt() const { return n_rt() + 1; }
    __device__ __forceinline__ const int32_t* grow(const struct BwdArgs& a) const;
    __device__ __forceinline__ int own_start(const struct BwdArgs& a) const;
};

__device__ __forceinline__ const int32_t* Item::grow(const BwdArgs& a) const { return a.gidx + (int64_t)u * a.wg; }
__device__ __forceinline__ int Item::own_start(const BwdArgs&) const { return own0; }

// Item `it` of the block path: a query block and a pair of its q-heads; of
// the strictly causal variant: a window of wu::kWin positions and four q-heads.
template <bool CAUSAL>
__device__ __forceinline__ void decode_item(const BwdArgs& a, int it, Item& m)
{
    if constexpr (CAUSAL) {
        const int n_y = (a.G + 3) / 4;
        m.u = it / n_y;
        m.head0 = 4 * (it % n_y);
        m.bg = m.u / int(a.nWin);
        m.w0 = (m.u % int(a.nWin)) * wu::kWin;
        m.qb = 0;
        m.own0 = int(64 * ((a.T_hist + m.w0) / 64));
    } else {
        const int n_pairs = (a.G + 1) / 2;
        m.u = it / n_pairs;
        m.head0 = 2 * (it % n_pairs);
        m.qb = m.u % int(a.nQB);
        m.bg = m.u / int(a.nQB);
        m.w0 = m.qb * 64;
        m.own0 = int(a.T_hist) + m.qb * 64;
    }
}

// Routed-group count n_g and segment-tile count n_seg of item `it`.  The
// routed groups are an ascending prefix of the index row: of the n_g, c_hist
// lie wholly in detached history (group j holds segment tokens iff
// 8 j >= T_hist), so the tiles from c_hist / 8 on, and the own chunk, hold
// segment keys.  Whole-warp call.
__device__ __forceinline__ int2 count_row(const BwdArgs& a, int64_t it, int lane)
{
    const int32_t* grow = a.gidx + (it / ((a.G + 1) / 2)) * a.wg;
    const int64_t first_seg_group = a.T_hist / 8;
    int n_g = 0, c_hist = 0;
    for (int base = 0; base < a.wg; base += 32) {
        const int i = base + lane;
        const int32_t j = i < a.wg ? __ldg(grow + i) : -1;
        n_g += __popc(__ballot_sync(0xFFFFFFFFu, j >= 0));
        c_hist += __popc(__ballot_sync(0xFFFFFFFFu, j >= 0 && j < first_seg_group));
    }
    const int n_rt = (n_g + 7) / 8;
    return make_int2(n_g, c_hist < n_g ? n_rt - c_hist / 8 + 1 : 1);
}

// Items a CTA decodes once, in its prologue, into shared memory; later ones
// (more than kItemTab items per CTA) are read and counted when reached.
constexpr int kItemTab = 64;

// Global index of CTA blockIdx.x's k-th item.
__device__ __forceinline__ int item_at(const BwdArgs& a, const int4* tab, int k)
{
    return k < kItemTab ? tab[k].x : __ldg(a.sched + (int64_t)k * gridDim.x + blockIdx.x);
}

// Item k of this CTA.  Whole-warp call.
template <bool CAUSAL>
__device__ __forceinline__ Item make_item(const BwdArgs& a, const int4* tab, int k, int lane)
{
    Item m;
    int it, n_g, n_seg;
    if (k < kItemTab) {
        const int4 e = tab[k];
        it = e.x;
        n_g = e.y;
        n_seg = e.z;
    } else {
        it = __ldg(a.sched + (int64_t)k * gridDim.x + blockIdx.x);
        const int2 c = count_row(a, it, lane);
        n_g = c.x;
        n_seg = c.y;
    }
    decode_item<CAUSAL>(a, it, m);
    m.n_g = n_g;
    m.n_seg = n_seg;
    return m;
}

// Persistent: CTA c processes the items of its column of the schedule, as
// many as round-robin would give it.  Barrier phases run on a global
// key-tile counter (gt), a segment-tile counter (gs) and an item counter (k)
// that every role advances identically.
// CAUSAL: the strictly causal variant, one window item per CTA (CTA c runs
// item sched[c], the items ordered heaviest first): its key tiles are the
// union of the window's routed groups (built in the prologue with the rows'
// sums D), rows are masked by their position's routing, and the K ring has
// 3 stages to make room for the union.
template <bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_k8, const __grid_constant__ CUtensorMap tm_v8,
                   const __grid_constant__ CUtensorMap tm_k64, const __grid_constant__ CUtensorMap tm_v64,
                   const __grid_constant__ CUtensorMap tm_dq, const BwdArgs a)
{
    constexpr int KST = CAUSAL ? 3 : kKStages;         // K stages
    constexpr int kHeads = CAUSAL ? 4 : 2;              // q-heads of the M-tile
    constexpr int kRows = 128 / kHeads;                 // query rows of each head
    using L = BwdSmem<KST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::bar_off;
    auto bar_q = [&](int b) { return bar0 + 8 * (kBarQ + b); };
    auto bar_kfull = [&](int s) { return bar0 + 8 * (kBarKFull + s); };
    auto bar_kempty = [&](int s) { return bar0 + 8 * (kBarKEmpty + s); };
    auto bar_vfull = [&](int s) { return bar0 + 8 * (kBarVFull + s); };
    auto bar_vempty = [&](int s) { return bar0 + 8 * (kBarVEmpty + s); };
    auto bar_sdp = [&](int b) { return bar0 + 8 * (kBarSdp + b); };
    auto bar_ps = [&](int b) { return bar0 + 8 * (kBarPs + b); };
    auto bar_sfree = [&](int b) { return bar0 + 8 * (kBarSfree + b); };   // dQ of the buffer's tile done
    const uint32_t bar_final_sdp = bar0 + 8 * kBarFinalSdp;
    const uint32_t bar_dsum = bar0 + 8 * kBarDsum;
    const uint32_t bar_kv = bar0 + 8 * kBarKv;
    const uint32_t bar_drained = bar0 + 8 * kBarDrained;
    const uint32_t bar_pfree = bar0 + 8 * kBarPfree;
    const uint32_t bar_qfree = bar0 + 8 * kBarQfree;
    const uint32_t bar_dqfree = bar0 + 8 * kBarDqfree;
    const uint32_t bar_final = bar0 + 8 * kBarFinal;
    const uint32_t bar_dqs_full = bar0 + 8 * kBarDqsFull;     // dQ staged in shared memory
    const uint32_t bar_dqs_free = bar0 + 8 * kBarDqsFree;     // its bulk stores have read it
    int4* tab = reinterpret_cast<int4*>(smem + L::tab_off);
    // Item k's Q/dO live in buffer k & 1, its P/dS in buffer (k + 1) & 1.
    auto xbuf = [&](int k) { return sbase + L::x_off + uint32_t(k & 1) * L::kX; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::tmem_slot_off);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n_mine = int((a.n_items - blockIdx.x + gridDim.x - 1) / gridDim.x);

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_q(b), 1);
            mbar_init(bar_sdp(b), 1);
            mbar_init(bar_ps(b), kCompute);
            mbar_init(bar_sfree(b), 1);
        }
        for (int s = 0; s < KST; ++s) {
            mbar_init(bar_kfull(s), 1);
            mbar_init(bar_kempty(s), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(bar_vfull(s), 1);
            mbar_init(bar_vempty(s), 1);
        }
        mbar_init(bar_kv, 1);
        mbar_init(bar_drained, kCompute);
        mbar_init(bar_pfree, 1);
        mbar_init(bar_qfree, 1);
        mbar_init(bar_dqfree, kCompute);
        mbar_init(bar_final, 1);
        mbar_init(bar_dqs_full, kCompute);
        mbar_init(bar_dqs_free, 1);
        mbar_init(bar_final_sdp, 1);
        mbar_init(bar_dsum, kCompute);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) tmem_alloc(smem_u32(tmem_slot), 512);
    // Setup above touches no global memory; the inputs are read from here on.
    pdl_wait();
    pdl_trigger();
    wu::View uv{};
    if constexpr (CAUSAL) {
        // The CTA's one item: the union of its window's routed groups and its
        // segment tiles.
        __shared__ int s_n, s_hist;
        const int it0 = int(chk::sched_item(a.sched));   // grid = items
        Item m0;
        decode_item<true>(a, it0, m0);
        uv = wu::view(smem + L::union_off, a.n_groups, a.wg);
        if (threadIdx.x == 0) s_hist = 0;
        const int n = wu::build(a.gidx + ((int64_t)m0.bg * a.T_seg + m0.w0) * a.wg, a.wg, m0.own0 / 8, uv, &s_n,
                                chk::kSiteCausalBwd);
        int c = 0;
        for (int k = threadIdx.x; k < n; k += kThreads) c += uv.list[k] < a.T_hist / 8;
        c = __reduce_add_sync(0xFFFFFFFFu, c);
        if (lane == 0 && c) atomicAdd(&s_hist, c);
        __syncthreads();
        if (threadIdx.x == 0) {
            const int n_rt = (n + 7) / 8, c_hist = s_hist;
            tab[0] = make_int4(it0, n, c_hist < n ? n_rt - c_hist / 8 + 1 : 1, 0);
        }
    } else {
        // Decode the CTA's first items (warp w: items w, w + 19, ...).
        const int n_tab = n_mine < kItemTab ? n_mine : kItemTab;
        for (int k = warp; k < n_tab; k += kThreads / 32) {
            const int32_t it = __ldg(a.sched + (int64_t)k * gridDim.x + blockIdx.x);
            const int2 c = count_row(a, it, lane);
            if (lane == 0) tab[k] = make_int4(it, c.x, c.y, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_do);
            prefetch_tmap(&tm_k8);
            prefetch_tmap(&tm_v8);
            prefetch_tmap(&tm_k64);
            prefetch_tmap(&tm_v64);
        }
        // Q / dO of item kq_ (lane 0) into buffer kq_ & 1, which held item
        // kq_-1's P / dS.
        auto load_q = [&](int kq_) {
            Item mq;
            decode_item<CAUSAL>(a, item_at(a, tab, kq_), mq);
            const int64_t b = mq.bg / a.Hkv, g = mq.bg % a.Hkv;
            mbar_expect_tx(bar_q(kq_ & 1), 2 * 2 * H * 64 * 128);
            for (int hp = 0; hp < kHeads; ++hp) {
                const int head = mq.head0 + hp;
                const int y = head < a.G ? int((b * a.Hq + g * a.G + head) * a.T_seg + mq.w0) : a.q_rows;
                for (int c = 0; c < H; ++c) {
                    const uint32_t off = c * L::kRows128 + hp * kRows * 128;
                    tma_load_2d(xbuf(kq_) + off, &tm_q, 64 * c, y, bar_q(kq_ & 1));
                    tma_load_2d(xbuf(kq_) + 2 * L::kRows128 + off, &tm_do, 64 * c, y, bar_q(kq_ & 1));
                }
                // Causal: the item's rows of O, read when its rows' sums D are formed.
                if (CAUSAL && head < a.G) bulk_prefetch_l2(a.O + (int64_t)y * a.d, uint32_t(kRows * a.d * 4));
            }
        };
        int last_k[KST], last_v[kVStages];              // last tile loaded per stage
        for (int j = 0; j < KST; ++j) last_k[j] = -1;
        for (int j = 0; j < kVStages; ++j) last_v[j] = -1;
        int q_issued = -1;                                  // last item whose Q / dO load was issued
        uint32_t gt = 0;
        bool ok = true;
        for (int k = 0; k < n_mine && ok; ++k) {
            const Item m = make_item<CAUSAL>(a, tab, k, lane);
            const int nt = m.nt(), n_rt = m.n_rt();
            const int32_t* grow = m.grow(a);
            const int64_t kv_base = (int64_t)m.bg * a.cap;
            for (int p = 0; p < nt && ok; ++p, ++gt) {
                const int t = nt - 1 - p;
                const int ks = gt % KST, vs = gt % kVStages;
                // Rows of the tile: lane l < 8 holds group slot l (a routed
                // tile) or lane 0 the own chunk's first row.
                int y = 0;
                if (t < n_rt) {
                    const int gi = t * 8 + lane;
                    if (lane < 8) {
                        int grp;
                        if constexpr (CAUSAL) grp = uv.list[gi < m.n_g ? gi : 0];   // checked when built
                        else grp = chk::group(__ldg(grow + (gi < m.n_g ? gi : 0)), m.own0 / 8, chk::kSiteBwdTcLoad);
                        y = int(kv_base + (int64_t)grp * 8);
                    }
                } else {
                    y = int(kv_base + m.own_start(a));
                }
                // K (or V) of the tile into stage `st` of `base`: 8-row
                // gathers, or the own chunk's two 64-row boxes.
                auto load_tile = [&](const CUtensorMap* m8, const CUtensorMap* m64, uint32_t dst, uint32_t bar) {
                    if (t < n_rt) {
                        if (lane < 8)
                            for (int c = 0; c < H; ++c) tma_load_2d(dst + c * L::kKVHalf + lane * 1024, m8, 64 * c, y, bar);
                    } else if (lane == 0) {
                        for (int c = 0; c < H; ++c) tma_load_2d(dst + c * L::kKVHalf, m64, 64 * c, y, bar);
                    }
                };
                if (lane == 0) {
                    // This item's Q / dO before any wait that their MMAs
                    // gate; the next item's as soon as this one's P / dS are
                    // released (tested without blocking).
                    if (q_issued < k) {
                        ok = k == 0 || mbar_wait(bar_pfree, (k - 1) & 1, kSitePfree);
                        if (ok) load_q(k);
                        q_issued = k;
                    }
                    if (ok && q_issued == k && k + 1 < n_mine && mbar_test(bar_pfree, k & 1)) {
                        load_q(k + 1);
                        q_issued = k + 1;
                    }
                    if (ok) ok = gt < KST || mbar_wait(bar_kempty(ks), ((gt / KST) - 1) & 1, kSiteEmpty);
                    if (ok) mbar_expect_tx(bar_kfull(ks), H * kKeys * 128);
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) break;
                last_k[ks] = gt;
                load_tile(&tm_k8, &tm_k64, sbase + L::k_off + ks * H * L::kKVHalf, bar_kfull(ks));
                __syncwarp();
                if (lane == 0) {
                    ok = gt < kVStages || mbar_wait(bar_vempty(vs), ((gt / kVStages) - 1) & 1, kSiteEmpty);
                    if (ok) mbar_expect_tx(bar_vfull(vs), H * kKeys * 128);
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) break;
                last_v[vs] = gt;
                load_tile(&tm_v8, &tm_v64, sbase + L::v_off + vs * H * L::kKVHalf, bar_vfull(vs));
                __syncwarp();
            }
        }
        // Wind down: every copy issued has landed before the CTA exits (the
        // Q / dO loads before the last one were read by MMAs pfree tracked).
        __syncwarp();
        if (lane == 0 && !ok) {
            for (int j = 0; j < KST; ++j)
                if (last_k[j] >= 0) mbar_wait(bar_kfull(j), (last_k[j] / KST) & 1, kSiteDrain);
            for (int j = 0; j < kVStages; ++j)
                if (last_v[j] >= 0) mbar_wait(bar_vfull(j), (last_v[j] / kVStages) & 1, kSiteDrain);
            if (q_issued >= 0) mbar_wait(bar_q(q_issued & 1), (q_issued >> 1) & 1, kSiteDrain);
        }
    } else if (warp == kSdpWarp) {
        // --------------------------------------------------- S / dP issuer
        // Tile g (the CTA's g-th key tile over all its items) writes S and
        // dP into buffer g & 1, which tile g - 2's dS still occupies until
        // that tile's dQ MMAs complete (sfree).
        constexpr uint32_t id_sdp = idesc_bf16(128, kKeys, 0, 0);
        bool ok = true;
        uint32_t g = 0;
        for (int k = 0; k < n_mine && ok; ++k) {
            const int nt = make_item<CAUSAL>(a, tab, k, lane).nt();
            for (int p = 0; p < nt && ok; ++p, ++g) {
                bool r = true;
                if (lane == 0) {
                    const int ks = g % KST, vs = g % kVStages, bb = g & 1;
                    if (p == 0) r = mbar_wait(bar_q(k & 1), (k >> 1) & 1, kSiteQ);
                    if (r && g >= 2) r = mbar_wait(bar_sfree(bb), ((g - 2) >> 1) & 1, kSiteSfree);
                    if (r) r = mbar_wait(bar_kfull(ks), (g / KST) & 1, kSiteFull);
                    if (r) r = mbar_wait(bar_vfull(vs), (g / kVStages) & 1, kSiteFull);
                    if (r) {
                        tc_fence_after();
                        // Descriptors of the operand bases; a K step adds its
                        // byte offset / 16 to the address field.
                        const uint32_t qa = xbuf(k);
                        const uint64_t dq = sdesc_sw128(qa, 16, 1024), ddo = sdesc_sw128(qa + 2 * L::kRows128, 16, 1024);
                        const uint64_t dk = sdesc_sw128(sbase + L::k_off + ks * H * L::kKVHalf, 16, 1024);
                        const uint64_t dv = sdesc_sw128(sbase + L::v_off + vs * H * L::kKVHalf, 16, 1024);
                        const uint32_t ts = tmem + kColS + bb * kKeys, tdp = tmem + kColDP + bb * kKeys;
#pragma unroll
                        for (int kk = 0; kk < 4 * H; ++kk) {
                            const uint32_t o = ((kk / 4) * L::kRows128 + (kk % 4) * 32) >> 4;
                            const uint32_t ko = ((kk / 4) * L::kKVHalf + (kk % 4) * 32) >> 4;
                            mma_ss(ts, dq + o, dk + ko, id_sdp, kk > 0);
                            mma_ss(tdp, ddo + o, dv + ko, id_sdp, kk > 0);
                        }
                        mma_commit(bar_sdp(bb));
                        mma_commit(bar_vempty(vs));                 // V is read by dP only
                    }
                }
                ok = __shfl_sync(0xFFFFFFFFu, r, 0);
            }
        }
        if (lane == 0) {
            // Every MMA issued here is complete before tensor memory is released.
            mma_commit(bar_final_sdp);
            mbar_wait(bar_final_sdp, 0, kSiteFinalSdp);
        }
    } else if (warp == kMmaWarp) {
        // --------------------------------------------------- gradient issuer
        constexpr uint32_t id_dq = idesc_bf16(128, D, 0, 1);        // dQ: A dS (tensor memory), B K MN-major
        constexpr uint32_t id_kv = idesc_bf16(128, kKeys, 1, 1);    // dV^T, dK^T: both MN-major
        bool ok = true;
        uint32_t gt = 0, gs = 0;
        for (int k = 0; k < n_mine && ok; ++k) {
            const Item mc = make_item<CAUSAL>(a, tab, k, lane);
            const int nt = mc.nt(), n_seg = mc.n_seg;
            for (int p = 0; ok && p < nt; ++p, ++gt) {
                const int ks = gt % KST, bb = gt & 1;
                const bool seg = p < n_seg;
                if (lane == 0) {
                    ok = mbar_wait(bar_ps(bb), (gt >> 1) & 1, kSitePs);
                    // dQ accumulates from zero: the previous item's dQ is read out.
                    if (ok && p == 0 && k > 0) ok = mbar_wait(bar_dqfree, (k - 1) & 1, kSiteDqfree);
                    if (ok) {
                        tc_fence_after();
                        // dQ += dS K, dS hi and lo from tensor memory (over S).
                        const uint64_t kb = sdesc_sw128(sbase + L::k_off + ks * H * L::kKVHalf, L::kKVHalf, 1024);
                        const uint32_t ds = tmem + kColS + bb * kKeys;
                        const bool acc = p > 0;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            mma_ts(tmem + kColDQ, ds + 16 * kk, kb + (kk * 2048 >> 4), id_dq, acc || kk > 0);
                            mma_ts(tmem + kColDQ, ds + 16 * kk + 8, kb + (kk * 2048 >> 4), id_dq, true);
                        }
                        mma_commit(bar_sfree(bb));                  // S / dP buffer bb reusable
                    }
                    if (ok && seg) {
                        // dV^T = dO^T P and dK^T = Q^T dS over the 128 query
                        // rows, once the previous segment tile's are read out.
                        if (gs >= 1) ok = mbar_wait(bar_drained, (gs - 1) & 1, kSiteDrained);
                        if (ok) {
                            tc_fence_after();
                            const uint32_t qa = xbuf(k), pa = xbuf(k + 1);
                            const uint64_t dOt = sdesc_sw128(qa + 2 * L::kRows128, L::kRows128, 1024);
                            const uint64_t Qt = sdesc_sw128(qa, L::kRows128, 1024);
                            const uint64_t Ph = sdesc_sw128(pa, L::kRows128, 1024);
                            const uint64_t Pl = sdesc_sw128(pa + L::kRows128, L::kRows128, 1024);
                            const uint64_t Sh = sdesc_sw128(pa + 2 * L::kRows128, L::kRows128, 1024);
                            const uint64_t Sl = sdesc_sw128(pa + 3 * L::kRows128, L::kRows128, 1024);
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint32_t o = (kk * 2048) >> 4;
                                mma_ss(tmem + kColDV, dOt + o, Ph + o, id_kv, kk > 0);
                                mma_ss(tmem + kColDV, dOt + o, Pl + o, id_kv, true);
                                mma_ss(tmem + kColDK, Qt + o, Sh + o, id_kv, kk > 0);
                                mma_ss(tmem + kColDK, Qt + o, Sl + o, id_kv, true);
                            }
                            mma_commit(bar_kv);
                            if (p == n_seg - 1) mma_commit(bar_pfree);   // P / dS no longer read
                        }
                    }
                    if (ok) {
                        mma_commit(bar_kempty(ks));                      // K read by S (done) and dQ
                        if (p == nt - 1) mma_commit(bar_qfree);          // Q / dO no longer read
                    }
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (seg) ++gs;
            }
        }
        if (lane == 0) {
            // Every MMA issued here is complete before tensor memory is released.
            mma_commit(bar_final);
            mbar_wait(bar_final, 0, kSiteFinal);
        }
    } else {
        // ------------- P and dS, then the dK / dV atomics and the dQ epilogue
        // Thread (warp w, lane l): query row r = 32*(w%4) + l of the M-tile
        // (its tensor-memory lane) and the 16-key quarter kq = w/4 of each tile.
        const int r = (warp % 4) * 32 + lane, kq = warp / 4;
        const int hp = r / kRows, qi = r % kRows;          // head within the tile, query within its rows
        const uint32_t lane_off = uint32_t((warp % 4) * 32) << 16;
        // First token of the quarter's two group slots of tile t (-64: padding).
        auto group_bases = [&](const Item& m, int t, int (&gb)[2]) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int gi = t * 8 + 2 * kq + q;
                int grp = -8;
                if (t != m.n_rt() && gi < m.n_g) {
                    if constexpr (CAUSAL) grp = uv.list[gi];
                    else grp = chk::group(__ldg(m.grow(a) + gi), m.own0 / 8, chk::kSiteBwdTcKeys);
                }
                gb[q] = t == m.n_rt() ? m.own_start(a) + 16 * kq + 8 * q : grp * 8;
            }
        };
        // dV^T / dK^T of a segment tile (d = tensor-memory lane r, keys of
        // quarter kq) added to the segment's rows; history keys and padding
        // are skipped.  Tensor memory is released before the atomics.
        auto dkv_epilogue = [&](int bg, const int (&gb)[2]) {
            tc_fence_after();
            uint32_t vv[16], kv[16];
            tmem_ld16(tmem + lane_off + kColDV + 16 * kq, vv);
            tmem_ld16(tmem + lane_off + kColDK + 16 * kq, kv);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar_drained);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int key = gb[j / 8] + j % 8;
                if (key < a.T_hist || r >= a.d) continue;   // padding, detached history, zero columns
                const int64_t o = ((int64_t)bg * a.T_seg + (key - a.T_hist)) * a.d + r;
                atomicAdd(a.dV + o, __uint_as_float(vv[j]));
                atomicAdd(a.dK + o, __uint_as_float(kv[j]) * a.scale);
            }
        };
        // Per-row constants of an item.
        struct RowInfo { int row, own_lim; bool ok; float lse2, Dr; };
        auto row_info = [&](const Item& m) {
            RowInfo ri;
            const int head = m.head0 + hp;
            ri.ok = head < a.G;
            const int b = m.bg / a.Hkv, g = m.bg % a.Hkv;
            ri.row = int((b * a.Hq + g * a.G + head) * a.T_seg) + m.w0 + qi;
            ri.own_lim = int(a.T_hist) + m.w0 + qi - m.own0;   // own-chunk keys 0 .. own_lim visible
            ri.lse2 = ri.ok ? __ldg(a.lse + ri.row) * kLog2e : 0.f;
            if constexpr (CAUSAL) ri.Dr = 0.f;                 // formed at the item's first tile
            else ri.Dr = ri.ok ? __ldg(a.Drow + ri.row) : 0.f;
            return ri;
        };
        uint32_t gt = 0, gs = 0;
        bool ok = true;
        Item m = make_item<CAUSAL>(a, tab, 0, lane);   // gridDim.x <= n_items
        RowInfo ri = row_info(m);
        for (int k = 0; k < n_mine && ok; ++k) {
            const bool row_ok = ri.ok;
            const int own_lim = ri.own_lim;
            const float lse2 = ri.lse2;
            float Dr = ri.Dr;
            const uint32_t pd = xbuf(k + 1) - sbase;        // this item's P / dS buffer
            uint8_t* prow_hi = smem + pd + r * 128;
            uint8_t* prow_lo = prow_hi + L::kRows128;
            uint8_t* srow_hi = prow_hi + 2 * L::kRows128;
            uint8_t* srow_lo = prow_hi + 3 * L::kRows128;
            int gb_prev[2] = {-64, -64};
            bool pending = false;                           // a segment tile's dK / dV are due
            const int nt = m.nt(), n_rt = m.n_rt();
            for (int p = 0; p < nt && ok; ++p, ++gt) {
                const int t = nt - 1 - p;
                const int bb = gt & 1;
                const bool seg = p < m.n_seg;
                int gb[2] = {-64, -64};
                if (seg) group_bases(m, t, gb);             // in flight during the tile
                ok = mbar_wait(bar_sdp(bb), (gt >> 1) & 1, kSiteSdp);
                if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
                tc_fence_after();
                if constexpr (CAUSAL) {
                    if (p == 0) {
                        // D = rowsum(dO * O) of row r: this thread's quarter kq of
                        // its row of O (prefetched into L2 with the item's Q / dO)
                        // and of the row of dO in shared memory (its load is
                        // complete: bar_q).  The four quarters meet in the dQ
                        // columns of tensor memory, free until the item's first dQ
                        // MMA (which waits for this tile's dS) once the previous
                        // item's dQ has been read out (dqfree).
                        ok = mbar_wait(bar_q(k & 1), (k >> 1) & 1, kSiteQ);
                        if (ok && k > 0) ok = mbar_wait(bar_dqfree, (k - 1) & 1, kSiteDqfree);
                        float part = 0.f;
                        if (row_ok && 32 * kq < a.d) {
                            float4 o4[8];
                            const float4* src = reinterpret_cast<const float4*>(a.O + (int64_t)ri.row * a.d + 32 * kq);
#pragma unroll
                            for (int j = 0; j < 8; ++j) o4[j] = __ldg(src + j);
                            const uint8_t* drow =
                                smem + (xbuf(k) - sbase) + 2 * L::kRows128 + (kq / 2) * L::kRows128 + r * 128;
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj) {
                                const int phys = ((kq % 2) * 4 + jj) ^ (r & 7);   // 128-byte swizzle
                                const uint4 w4 = *reinterpret_cast<const uint4*>(drow + phys * 16);
                                const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
                                const float4 oa = o4[2 * jj], ob = o4[2 * jj + 1];
                                const float of[8] = {oa.x, oa.y, oa.z, oa.w, ob.x, ob.y, ob.z, ob.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    part = fmaf(__uint_as_float(w[e] << 16), of[2 * e], part);
                                    part = fmaf(__uint_as_float(w[e] & 0xFFFF0000u), of[2 * e + 1], part);
                                }
                            }
                        }
                        tmem_st1(tmem + lane_off + kColDQ + kq, __float_as_uint(part));
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(bar_dsum);
                        if (ok) ok = mbar_wait(bar_dsum, k & 1, kSiteDsum);
                        if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
                        tc_fence_after();
                        uint32_t dp[4];
                        tmem_ld4(tmem + lane_off + kColDQ, dp);
                        tmem_wait_ld();
                        Dr = row_ok ? (__uint_as_float(dp[0]) + __uint_as_float(dp[1])) +
                                          (__uint_as_float(dp[2]) + __uint_as_float(dp[3]))
                                    : 0.f;
                    }
                }
                const bool own = t == n_rt;
                uint32_t sr[16], pr[16];
                tmem_ld16(tmem + lane_off + kColS + bb * kKeys + 16 * kq, sr);
                tmem_ld16(tmem + lane_off + kColDP + bb * kKeys + 16 * kq, pr);
                tmem_wait_ld();
                uint32_t ph[8], pl[8], dsw[16];             // dsw: dS hi (8), then dS lo (8)
                // Every key of a full routed tile is valid for every row (block
                // path): no masks there; partial tiles and the own chunk mask keys.
                const bool full = !CAUSAL && row_ok && !own && t * 8 + 8 <= m.n_g;
                // Causal: the masks of the quarter's two group slots of the tile.
                uint32_t mw[2] = {0u, 0u};
                if constexpr (CAUSAL) {
                    if (!own) {
#pragma unroll
                        for (int q2 = 0; q2 < 2; ++q2) {
                            const int slot = t * 8 + 2 * kq + q2;
                            mw[q2] = slot < m.n_g ? uv.mask[slot] : 0u;
                        }
                    }
                }
                const float2 c2 = make_float2(a.scale_log2, a.scale_log2);
                const float2 l2 = make_float2(-lse2, -lse2), d2 = make_float2(-Dr, -Dr);
#pragma unroll
                for (int j2 = 0; j2 < 8; ++j2) {
                    const int j0 = 16 * kq + 2 * j2;
                    const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[2 * j2]), __uint_as_float(sr[2 * j2 + 1])),
                                                c2, l2);
                    float2 pv = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                    if (!full) {
                        bool v0, v1;
                        if (own) {
                            v0 = j0 <= own_lim;
                            v1 = j0 + 1 <= own_lim;
                        } else if constexpr (CAUSAL) {
                            v0 = v1 = (mw[j2 / 4] >> qi) & 1u;   // keys j0, j0 + 1: one group
                        } else {
                            v0 = t * 8 + j0 / 8 < m.n_g;
                            v1 = t * 8 + (j0 + 1) / 8 < m.n_g;
                        }
                        v0 = v0 && row_ok;
                        v1 = v1 && row_ok;
                        pv.x = v0 ? pv.x : 0.f;
                        pv.y = v1 ? pv.y : 0.f;
                    }
                    const float2 ds = __fmul2_rn(
                        pv, __fadd2_rn(make_float2(__uint_as_float(pr[2 * j2]), __uint_as_float(pr[2 * j2 + 1])), d2));
                    split_bf16x2(ds.x, ds.y, dsw[j2], dsw[8 + j2]);
                    if (seg) split_bf16x2(pv.x, pv.y, ph[j2], pl[j2]);
                }
                // dS over this quarter's S columns: hi for keys 16kq.. at
                // column 16kq, lo at 16kq + 8 (the dQ MMA's A operand).
                tmem_st16(tmem + lane_off + kColS + bb * kKeys + 16 * kq, dsw);
                if (seg) {
                    // The previous segment tile's dK / dV MMAs read P / dS
                    // from this buffer (the item's first segment tile reuses
                    // the previous item's Q / dO, released at its end).
                    if (p > 0) {
                        ok = mbar_wait(bar_kv, (gs - 1) & 1, kSiteKv);
                        if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
                    } else if (k > 0) {
                        // The previous item's dQ boxes, staged here, have
                        // been read by their bulk stores.
                        if (threadIdx.x == 0) {
                            bulk_wait_read();
                            mbar_arrive(bar_dqs_free);
                        }
                        ok = mbar_wait(bar_dqs_free, (k - 1) & 1, kSiteDqs);
                        if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
                    }
                    // Row r, 16-byte chunk c lives at chunk c ^ (r % 8) (128-byte swizzle).
#pragma unroll
                    for (int c2i = 0; c2i < 2; ++c2i) {
                        const int pc = ((2 * kq + c2i) ^ (r & 7)) * 16;
                        *reinterpret_cast<uint4*>(srow_hi + pc) =
                            make_uint4(dsw[4 * c2i], dsw[4 * c2i + 1], dsw[4 * c2i + 2], dsw[4 * c2i + 3]);
                        *reinterpret_cast<uint4*>(srow_lo + pc) =
                            make_uint4(dsw[8 + 4 * c2i], dsw[9 + 4 * c2i], dsw[10 + 4 * c2i], dsw[11 + 4 * c2i]);
                        *reinterpret_cast<uint4*>(prow_hi + pc) =
                            make_uint4(ph[4 * c2i], ph[4 * c2i + 1], ph[4 * c2i + 2], ph[4 * c2i + 3]);
                        *reinterpret_cast<uint4*>(prow_lo + pc) =
                            make_uint4(pl[4 * c2i], pl[4 * c2i + 1], pl[4 * c2i + 2], pl[4 * c2i + 3]);
                    }
                    fence_async_smem();
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_ps(bb));
                // While this tile's MMAs run: the previous segment tile's dK / dV.
                if (pending) {
                    if (!seg) {
                        ok = mbar_wait(bar_kv, (gs - 1) & 1, kSiteKv);
                        if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
                    }
                    dkv_epilogue(m.bg, gb_prev);
                    pending = false;
                }
                if (seg) {
                    gb_prev[0] = gb[0];
                    gb_prev[1] = gb[1];
                    pending = true;
                    ++gs;
                }
            }
            if (!ok) break;
            // The next item's index row and row constants load meanwhile.
            const Item m_next = k + 1 < n_mine ? make_item<CAUSAL>(a, tab, k + 1, lane) : m;
            const RowInfo ri_next = row_info(m_next);
            if (pending) {
                ok = mbar_wait(bar_kv, (gs - 1) & 1, kSiteKv);
                if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
                dkv_epilogue(m.bg, gb_prev);
            }
            // dQ (times the softmax scale), columns 32kq.. of row r: into
            // this item's Q / dO buffer (free once its last MMAs completed) as
            // eight 64-row x 32-column boxes in the 128-byte-swizzled layout
            // of the dQ tensor map; thread 0 stores the boxes with bulk copies
            // that run on while the next item starts.  (Stores straight from
            // registers measured slower.)
            ok = mbar_wait(bar_qfree, k & 1, kSiteQfree);
            if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
            tc_fence_after();
            {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + kColDQ + 32 * kq, v);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(bar_dqfree);
                uint8_t* box = smem + (xbuf(k) - sbase) + (hp * 4 + kq) * (kRows * 128) + qi * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<float4*>(box + ((j ^ (qi & 7)) * 16)) =
                        make_float4(__uint_as_float(v[4 * j]) * a.scale, __uint_as_float(v[4 * j + 1]) * a.scale,
                                    __uint_as_float(v[4 * j + 2]) * a.scale, __uint_as_float(v[4 * j + 3]) * a.scale);
                fence_async_smem();
                mbar_arrive(bar_dqs_full);
            }
            if (threadIdx.x == 0) {
                ok = mbar_wait(bar_dqs_full, k & 1, kSiteDqs);
                if (ok) {
                    const int b = m.bg / a.Hkv, g = m.bg % a.Hkv;
                    for (int h2 = 0; h2 < kHeads; ++h2) {
                        const int head = m.head0 + h2;
                        if (head >= a.G) continue;           // no such head: nothing to store
                        const int y = int((b * a.Hq + g * a.G + head) * a.T_seg) + m.w0;
                        for (int c = 0; c < a.d / 32; ++c)
                            tma_store_2d(&tm_dq, 32 * c, y, xbuf(k) + (h2 * 4 + c) * (kRows * 128));
                    }
                    bulk_commit();
                }
            }
            if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
            m = m_next;
            ri = ri_next;
        }
        // The dQ bulk stores are complete (and have read shared memory)
        // before the CTA exits.
        if (threadIdx.x == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- schedule
// The backward kernel is persistent: its G CTAs take R = ceil(n / G) or R-1
// items each.  An item's time grows with its key tiles and, more steeply,
// with its segment tiles (their dK / dV products and atomics), which
// depend on the routing.  Round-robin lets a CTA with R items draw heavy
// ones and end well after the rest, so block 0 of the row-dot launch ranks
// the items by estimated cost, heaviest first (ties by index), and deals
// them out: the heaviest to the G - E CTAs that take R - 1 items, the
// lightest to the E that take R, in rounds whose direction alternates.
// sched[k * G + c] is CTA c's k-th item; CTA c takes the same number of
// items as under round-robin.  Only when a CTA takes at most kDealRounds
// items: with more, one item is a small part of a CTA's time, and the
// round-robin order, whose concurrent items are neighbouring blocks of the
// same (batch, kv-head) sharing K / V rows in L2, measured faster (B 4,
// 14 items a CTA: 2-7 % on the backward), so sched is then the identity.
constexpr int kCostClasses = 64;
constexpr int kDealRounds = 4;
constexpr int kMaxDealItems = 1024;

struct SchedArgs {
    const int32_t* gidx;
    int32_t* sched;
    int64_t n_items, first_seg_group;
    int n_pairs, wg, G;
};

// Estimated cost of item `it`: key tiles plus segment tiles (each of those
// costs about two), clamped to the class range.  Counts as count_row does,
// one thread per item.
__device__ __forceinline__ int item_cost(const SchedArgs& sa, int64_t it)
{
    const int32_t* row = sa.gidx + (it / sa.n_pairs) * sa.wg;
    int n_g = 0, c_hist = 0;
    if ((sa.wg & 3) == 0) {
        for (int i = 0; i < sa.wg; i += 4) {
            const int4 v = __ldg(reinterpret_cast<const int4*>(row + i));
            const int j[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                n_g += j[q] >= 0;
                c_hist += j[q] >= 0 && j[q] < sa.first_seg_group;
            }
        }
    } else {
        for (int i = 0; i < sa.wg; ++i) {
            const int32_t j = __ldg(row + i);
            n_g += j >= 0;
            c_hist += j >= 0 && j < sa.first_seg_group;
        }
    }
    const int n_rt = (n_g + 7) / 8;
    const int n_seg = c_hist < n_g ? n_rt - c_hist / 8 + 1 : 1;
    return min(n_rt + 1 + n_seg, kCostClasses - 1);
}

// Whole-block call (256 threads): counting sort of the items by cost class,
// stable within a class, then the deal described above.
__device__ void build_schedule(const SchedArgs& sa)
{
    __shared__ int hist[kCostClasses], next[kCostClasses];
    __shared__ int wcnt[8][kCostClasses];
    // Cost classes of the first kMaxDealItems items, read from the index
    // rows once (the deal runs for at most kDealRounds items a CTA: 592
    // items on 148 SMs); classes past it are recomputed.
    __shared__ uint8_t cls[kMaxDealItems];
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int64_t n = sa.n_items;
    if ((n + sa.G - 1) / sa.G > kDealRounds) {
        for (int64_t i = tid; i < n; i += 256) sa.sched[i] = int32_t(i);
        return;
    }
    for (int c = tid; c < kCostClasses; c += 256) hist[c] = 0;
    __syncthreads();
    for (int64_t i = tid; i < n; i += 256) {
        const int c = item_cost(sa, i);
        if (i < kMaxDealItems) cls[i] = uint8_t(c);
        atomicAdd(&hist[c], 1);
    }
    __syncthreads();
    // next[c] = items of classes above c (heaviest first): lane L sums
    // classes 2L and 2L + 1, a suffix scan over the lanes does the rest.
    if (warp == 0) {
        const int h0 = hist[2 * lane], h1 = hist[2 * lane + 1];
        const int own = h0 + h1;
        int suf = own;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_down_sync(0xFFFFFFFFu, suf, o);
            if (lane + o < 32) suf += v;
        }
        next[2 * lane + 1] = suf - own;
        next[2 * lane] = suf - own + h1;
    }
    __syncthreads();
    const int64_t G = sa.G, R = (n + G - 1) / G, E = n - (R - 1) * G, S = (G - E) * (R - 1);
    const uint32_t lt = (1u << lane) - 1u;
    for (int64_t base = 0; base < n; base += 256) {
        const int64_t i = base + tid;
        const int c = i >= n ? -1 : i < kMaxDealItems ? int(cls[i]) : item_cost(sa, i);
        for (int j = tid; j < 8 * kCostClasses; j += 256) (&wcnt[0][0])[j] = 0;
        __syncthreads();
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, c);
        const int below = __popc(peers & lt);
        if (c >= 0 && below == 0) wcnt[warp][c] = __popc(peers);
        __syncthreads();
        if (c >= 0) {
            int64_t rank = next[c] + below;
            for (int w = 0; w < warp; ++w) rank += wcnt[w][c];
            // Rank -> (CTA, round): ranks below S go to the CTAs E.. G-1
            // (R - 1 items), the rest to CTAs 0 .. E-1 (R items).
            const int64_t m = rank < S ? G - E : E, r = rank < S ? rank : rank - S;
            const int64_t round = r / m;
            int64_t pos = r % m;
            if (round & 1) pos = m - 1 - pos;
            const int64_t cta = rank < S ? E + pos : pos;
            sa.sched[round * G + cta] = int32_t(i);
        }
        __syncthreads();
        if (tid < kCostClasses) {
            int add = 0;
            for (int w = 0; w < 8; ++w) add += wcnt[w][tid];
            next[tid] += add;
        }
        __syncthreads();
    }
}

// D_row = sum_e dO[row][e] * O[row][e]: one warp per four rows, whose
// 16-byte loads of O and 8-byte loads of dO are all issued before the sums.
// The same launch zeroes dK_seg and dV_seg (the backward kernel adds into
// them), n4 float4s each, grid-stride; its block 0 builds the backward's
// item schedule instead.
constexpr int kRowdotRows = 4;

template <int DH>
__global__ void __launch_bounds__(256)
rowdot_kernel(const float* __restrict__ O, const __nv_bfloat16* __restrict__ dO, float* __restrict__ Drow,
              int64_t rows, float4* __restrict__ dK, float4* __restrict__ dV, int64_t n4, const SchedArgs sa)
{
    pdl_wait();
    pdl_trigger();
    if (blockIdx.x == 0) {
        build_schedule(sa);
        return;
    }
    const int64_t bx = blockIdx.x - 1;
    const int64_t tid = bx * blockDim.x + threadIdx.x;
    const int64_t nthreads = (int64_t)(gridDim.x - 1) * blockDim.x;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t j = tid; j < n4; j += nthreads) {
        dK[j] = z;
        dV[j] = z;
    }
    const int64_t row0 = (bx * 8 + threadIdx.x / 32) * kRowdotRows;
    const int lane = threadIdx.x & 31;
    float acc[kRowdotRows];
    if constexpr (DH == 128) {          // a lane: 4 columns (16 bytes of O, 8 of dO)
        float4 o[kRowdotRows];
        uint2 w[kRowdotRows];
#pragma unroll
        for (int q = 0; q < kRowdotRows; ++q) {
            const int64_t row = row0 + q;
            o[q] = row < rows ? __ldg(reinterpret_cast<const float4*>(O + row * DH) + lane) : z;
            w[q] = row < rows ? __ldg(reinterpret_cast<const uint2*>(dO + row * DH) + lane) : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < kRowdotRows; ++q)
            acc[q] = o[q].x * __uint_as_float(w[q].x << 16) + o[q].y * __uint_as_float(w[q].x & 0xFFFF0000u) +
                     o[q].z * __uint_as_float(w[q].y << 16) + o[q].w * __uint_as_float(w[q].y & 0xFFFF0000u);
    } else {                            // d = 64: 2 columns a lane
        float2 o[kRowdotRows];
        uint32_t w[kRowdotRows];
#pragma unroll
        for (int q = 0; q < kRowdotRows; ++q) {
            const int64_t row = row0 + q;
            o[q] = row < rows ? __ldg(reinterpret_cast<const float2*>(O + row * DH) + lane) : make_float2(0.f, 0.f);
            w[q] = row < rows ? __ldg(reinterpret_cast<const uint32_t*>(dO + row * DH) + lane) : 0u;
        }
#pragma unroll
        for (int q = 0; q < kRowdotRows; ++q)
            acc[q] = o[q].x * __uint_as_float(w[q] << 16) + o[q].y * __uint_as_float(w[q] & 0xFFFF0000u);
    }
#pragma unroll
    for (int q = 0; q < kRowdotRows; ++q) {
        const float v = warp_sum(acc[q]);
        if (lane == 0 && row0 + q < rows) Drow[row0 + q] = v;
    }
}

}  // namespace

int attn_bwd_tc_status(bool clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, sm100::g_status, sizeof v) != cudaSuccess) return -1;
    if (clear && v) {
        const int z = 0;
        cudaMemcpyToSymbol(sm100::g_status, &z, sizeof z);
    }
    return v;
}

bool attn_bwd_tc_supported(const Shape& s)
{
    const uint64_t q_rows = (uint64_t)s.B * s.Hq * s.T_seg, kv_rows = (uint64_t)s.B * s.Hkv * s.cap;
    return s.dtype == HGA_BF16 && (s.d == 64 || s.d == 128) && q_rows < (1ull << 31) && kv_rows < (1ull << 31) &&
           tensor_maps_available();
}

cudaError_t launch_attn_bwd_tc(const Shape& s, const void* Q, const void* K, const void* V, const float* O,
                               const float* lse, const void* dO, const int32_t* gidx, float* dQ,
                               float* dK_seg, float* dV_seg, float* Drow, cudaStream_t st)
{
    const int64_t rows = (int64_t)s.B * s.Hq * s.T_seg;
    const int64_t n4 = (int64_t)s.B * s.Hkv * s.T_seg * s.d / 4;   // d = 64 or 128: whole float4s
    const int64_t n_items = bwd_items(s);
    const int64_t grid = std::min<int64_t>(n_items, sm_count());
    // The scratch holds the row sums, then the schedule (Drow + rows).
    int32_t* sched = reinterpret_cast<int32_t*>(Drow + rows);
    SchedArgs sa;
    sa.gidx = gidx;
    sa.sched = sched;
    sa.n_items = n_items;
    sa.first_seg_group = s.T_hist / 8;
    sa.n_pairs = (s.G + 1) / 2;
    sa.wg = s.wg;
    sa.G = (int)grid;
    const int64_t rows_per_cta = 8 * kRowdotRows;
    auto rowdot = s.d == 128 ? rowdot_kernel<128> : rowdot_kernel<64>;
    cudaError_t e = launch_pdl(rowdot, dim3((unsigned)(1 + (rows + rows_per_cta - 1) / rows_per_cta)),
                               dim3(256), 0, st, O, static_cast<const __nv_bfloat16*>(dO), Drow, rows,
                               reinterpret_cast<float4*>(dK_seg), reinterpret_cast<float4*>(dV_seg), n4, sa);
    if (e != cudaSuccess) return e;
    CUtensorMap tq, tdo, tk8, tv8, tk64, tv64, tdq;
    const uint64_t q_rows = (uint64_t)rows, kv_rows = (uint64_t)s.B * s.Hkv * s.cap;
    // Maps of the tensors' own width d: boxes past it (d = 64) read zeros.
    if (!make_bf16_map(&tq, Q, q_rows, s.d, 64) || !make_bf16_map(&tdo, dO, q_rows, s.d, 64) ||
        !make_bf16_map(&tk8, K, kv_rows, s.d, 8) || !make_bf16_map(&tv8, V, kv_rows, s.d, 8) ||
        !make_bf16_map(&tk64, K, kv_rows, s.d, 64) || !make_bf16_map(&tv64, V, kv_rows, s.d, 64) ||
        !make_f32_map(&tdq, dQ, q_rows, s.d, 64))
        return cudaErrorInvalidValue;
    BwdArgs a{};
    a.gidx = gidx;
    a.lse = lse;
    a.Drow = Drow;
    a.O = O;
    a.dO = static_cast<const __nv_bfloat16*>(dO);
    a.dQ = dQ;
    a.dK = dK_seg;
    a.dV = dV_seg;
    a.Hq = s.Hq;
    a.Hkv = s.Hkv;
    a.G = s.G;
    a.wg = s.wg;
    a.d = s.d;
    a.T_hist = s.T_hist;
    a.T_seg = s.T_seg;
    a.nQB = s.nQB;
    a.cap = s.cap;
    a.q_rows = (int)q_rows;
    a.scale = s.scale;
    a.scale_log2 = s.scale * kLog2e;
    const int smem = BwdSmem<kKStages>::alloc;
    if ((e = cudaFuncSetAttribute(attn_bwd_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
        return e;
    a.n_items = n_items;
    a.sched = sched;
    return launch_pdl(attn_bwd_tc_kernel<false>, dim3((unsigned)grid), dim3(kThreads), (size_t)smem, st, tq, tdo,
                      tk8, tv8, tk64, tv64, tdq, a);
}

// Strictly causal variant: bf16, index rows of at most 64 groups (a window's
// union of at most 2048), shared memory permitting.
bool attn_bwd_tc_causal_supported(const Shape& s)
{
    const size_t smem = (size_t)BwdSmem<3>::union_off + wu::bytes(s.nG, s.wg) + 1024;
    return attn_bwd_tc_supported(s) && s.wg <= 64 && s.T_seg % wu::kWin == 0 && smem <= 227 * 1024;
}

cudaError_t launch_attn_bwd_tc_causal(const Shape& s, const void* Q, const void* K, const void* V, const float* O,
                                      const float* lse, const void* dO, const int32_t* gidx,
                                      const int32_t* sched, float* dQ, float* dK_seg, float* dV_seg,
                                      cudaStream_t st)
{
    // dK / dV accumulate with atomics: zeroed first.
    const size_t seg_bytes = sizeof(float) * (size_t)s.B * s.Hkv * s.T_seg * s.d;
    cudaError_t e = cudaMemsetAsync(dK_seg, 0, seg_bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dV_seg, 0, seg_bytes, st);
    if (e != cudaSuccess) return e;
    CUtensorMap tq, tdo, tk8, tv8, tk64, tv64, tdq;
    const uint64_t q_rows = (uint64_t)s.B * s.Hq * s.T_seg, kv_rows = (uint64_t)s.B * s.Hkv * s.cap;
    if (!make_bf16_map(&tq, Q, q_rows, s.d, wu::kWin) || !make_bf16_map(&tdo, dO, q_rows, s.d, wu::kWin) ||
        !make_bf16_map(&tk8, K, kv_rows, s.d, 8) || !make_bf16_map(&tv8, V, kv_rows, s.d, 8) ||
        !make_bf16_map(&tk64, K, kv_rows, s.d, 64) || !make_bf16_map(&tv64, V, kv_rows, s.d, 64) ||
        !make_f32_map(&tdq, dQ, q_rows, s.d, wu::kWin))
        return cudaErrorInvalidValue;
    BwdArgs a{};
    a.gidx = gidx;
    a.sched = sched;                 // CTA x runs item sched[x] (null: item x)
    a.Drow = nullptr;
    a.lse = lse;
    a.dQ = dQ;
    a.dK = dK_seg;
    a.dV = dV_seg;
    a.Hq = s.Hq;
    a.Hkv = s.Hkv;
    a.G = s.G;
    a.wg = s.wg;
    a.d = s.d;
    a.T_hist = s.T_hist;
    a.T_seg = s.T_seg;
    a.nQB = s.nQB;
    a.cap = s.cap;
    a.nWin = s.T_seg / wu::kWin;
    a.n_groups = s.nG;
    a.O = O;
    a.dO = static_cast<const __nv_bfloat16*>(dO);
    a.q_rows = (int)q_rows;
    a.scale = s.scale;
    a.scale_log2 = s.scale * kLog2e;
    // One window item per CTA (grid = items; the kernel's item loop runs once).
    a.n_items = (int64_t)s.B * s.Hkv * a.nWin * ((s.G + 3) / 4);
    const int smem = int((size_t)BwdSmem<3>::union_off + wu::bytes(s.nG, s.wg) + 1024);
    if ((e = cudaFuncSetAttribute(attn_bwd_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
        return e;
    return launch_pdl(attn_bwd_tc_kernel<true>, dim3((unsigned)a.n_items), dim3(kThreads), (size_t)smem, st, tq, tdo,
                      tk8, tv8, tk64, tv64, tdq, a);
}

// Check word of this translation unit's bounds checks (checked builds).
HGA_CHECK_WORD_READER(check_word_attn_tc_bwd)

}  // namespace hga
