// attn_tc_fwd.cu -- a5 routed attention forward on the tcgen05 tensor cores
// (bf16 inputs, float32 accumulation and softmax).
//
// Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com),
// section "What HGA does differently": after routing, only the exact token
// K/V of the selected groups is loaded for the attention; summaries are never
// attended.  Query i of a block also attends its own chunk up to itself.
//
// One CTA owns one (batch, kv-head, query block) and a pair of its q-heads:
// their two 64-query blocks stacked into one M-tile of 128 rows.  The CTAs of
// one query block are adjacent in the grid, so they run together and share
// the key tiles through L2.  Key tiles are 64 tokens: 8 routed groups (8 rows
// each, one TMA box per group and 64-column half of d) or the own chunk (one
// box).  Per key tile:
//     S  = Q K^T            tcgen05.mma  A = Q (smem), B = K (smem) -> TMEM
//     P  = exp2(S*c - m)    softmax warps, P -> TMEM over S as two bf16 parts
//                           hi + lo (P to ~14 bits)
//     O += P V              tcgen05.mma  A = P hi, P lo (TMEM), B = V (smem)
// The running maximum is only moved when a row's maximum grows by more than
// 2^8 (then O is rescaled in TMEM); any fixed reference point gives the same
// O / l, and it spares most rescales.
//
// Warp roles (320 threads): warps 0-7 softmax, warp w on rows 32(w%4).. of
// the M-tile (its tensor-memory lane quadrant) and keys 32(w/4).. of each
// tile; the two warps of a quadrant exchange their row maxima through shared
// memory once per tile.  Warp 8 is the TMA producer, warp 9 the tensor-memory
// owner and MMA issuer.  Tensor memory (256 columns): O (D columns) and two
// S/P buffers of 64 columns, so that S of the next key tile is computed while
// the softmax works on the current one.  With 97 KB of shared memory and 256
// columns, two CTAs share an SM: one's prologue and epilogue overlap the
// other's key loop.
#include <algorithm>

#include "check.cuh"
#include "hga_internal.cuh"
#include "router_core.cuh"
#include "sm100.cuh"
#include "window_union.cuh"

namespace hga {

namespace {

using namespace sm100;

constexpr int kKeys = 64;           // keys per tile
constexpr int kStages = 2;          // K tiles and V tiles in flight (separate rings)
constexpr int kSoftmaxWarps = 8;
constexpr int kSoftmax = 32 * kSoftmaxWarps;
constexpr int kProducerWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;
constexpr int kThreads = 32 * (kSoftmaxWarps + 2);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;

// Status codes of the bounded waits (site of the wait that ran out).
enum : int {
    kSiteQ = 101, kSiteFull, kSiteEmpty, kSiteS, kSiteP, kSiteO, kSiteFinal, kSiteDrain, kSiteStage, kSiteMax
};

template <int D>
struct FwdSmem {
    static constexpr int H = D / 64;                  // 64-column halves of d
    static constexpr uint32_t kTmemCols = 256;        // O (D) + S/P (2 x 64)
    static constexpr int kQTile = 128 * 128;          // one 64-column half: 128 rows x 128 B
    static constexpr int kKVHalf = kKeys * 128;       // 64 keys x 128 B
    static constexpr int q_off = 0;
    static constexpr int k_off = q_off + H * kQTile;
    static constexpr int v_off = k_off + kStages * H * kKVHalf;
    static constexpr int xmax_off = v_off + kStages * H * kKVHalf;   // float [2][4][2][32]
    static constexpr int bar_off = xmax_off + 2 * 4 * 2 * 32 * 4;
    // barriers: q, kfull[S], kempty[S], vfull[S], vempty[S], s[2], p[2], o[2],
    // final, stage, mx[2][4]
    static constexpr int n_bars = 1 + 4 * kStages + 2 + 2 + 2 + 2 + 8;
    static constexpr int tmem_slot_off = bar_off + 8 * n_bars;
    static constexpr int bytes = tmem_slot_off + 16;
    static constexpr int alloc = bytes + 1024;        // room to align the base to 1 KB
    // Strictly causal variant: the window's union of routed groups follows.
    static constexpr int union_off = (bytes + 15) & ~15;
    // The O stage of the epilogue (128 rows x D floats) reuses Q and K/V.
    static_assert(128 * D * 4 <= xmax_off, "O stage");
};

struct FwdArgs {
    const int32_t* gidx;
    float* O;
    float* lse;
    int Hq, Hkv, G, wg;
    int64_t T_hist, T_seg, nQB;
    int64_t nWin;        // strictly causal variant: windows of wu::kWin positions per (b, g)
    int64_t n_groups;    // groups of the context (T / 8): bounds the union's bitmap
    int q_rows;          // B*Hq*T_seg (rows of the Q map)
    int kv_rows;         // B*Hkv*cap (rows of the K / V maps)
    int64_t cap;         // K / V rows per (batch, kv-head)
    float scale_log2;
    const int32_t* sched;  // strictly causal variant: CTA x runs item sched[x] (null: item x)
};

// One M-tile of the forward: query block (or causal window) u and q-heads
// head0 .. head0 + kHeads - 1; grow is the block's index row.  The whole CTA
// calls it; it sets up its barriers and tensor memory, runs the tile and
// releases both, so a CTA may run several tiles one after another.
// CAUSAL: the strictly causal variant.  A CTA then owns wu::kWin
// neighbouring query positions of one (batch, kv-head) and four of its
// q-heads (row r: head r / 32, position r % 32 of the window); its key tiles
// are the union of the positions' routed groups, built in shared memory, and
// every row keeps only the groups its own position routed (a bit of the
// group's mask) plus its own chunk up to itself.  Q boxes are 32 rows.
// ROUTED: the fused route + forward kernel's tiles; grow is in shared memory.
template <int D, bool CAUSAL, bool ROUTED>
__device__ __forceinline__ void fwd_tile(const CUtensorMap* tm_q, const CUtensorMap* tm_k8, const CUtensorMap* tm_v8,
                                         const CUtensorMap* tm_k64, const CUtensorMap* tm_v64, const FwdArgs& a,
                                         const int64_t u, const int head0, const int32_t* grow)
{
    using L = FwdSmem<D>;
    constexpr int H = L::H;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::bar_off;
    const uint32_t bar_q = bar0;
    // Ring r (0 = K, 1 = V): full and empty barriers of its stages.
    auto bar_full = [&](int r, int s) { return bar0 + 8 * (1 + 2 * kStages * r + s); };
    auto bar_empty = [&](int r, int s) { return bar0 + 8 * (1 + 2 * kStages * r + kStages + s); };
    auto bar_s = [&](int b) { return bar0 + 8 * (1 + 4 * kStages + b); };
    auto bar_p = [&](int b) { return bar0 + 8 * (3 + 4 * kStages + b); };
    auto bar_o = [&](int b) { return bar0 + 8 * (5 + 4 * kStages + b); };
    const uint32_t bar_final = bar0 + 8 * (7 + 4 * kStages);
    const uint32_t bar_stage = bar0 + 8 * (8 + 4 * kStages);
    auto bar_mx = [&](int b, int q) { return bar0 + 8 * (9 + 4 * kStages + 4 * b + q); };
    float* xmax = reinterpret_cast<float*>(smem + L::xmax_off);   // [parity][quadrant][half][lane]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::tmem_slot_off);
    __shared__ int s_abort;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    constexpr int kHeads = CAUSAL ? 4 : 2;                  // q-heads of the M-tile
    constexpr int kRows = 128 / kHeads;                     // query rows of each head
    int64_t bg, w0, c0;                                     // first query of the tile; own chunk
    if constexpr (CAUSAL) {
        bg = u / a.nWin;
        w0 = (u % a.nWin) * wu::kWin;
        c0 = (a.T_hist + w0) / 64;
    } else {
        bg = u / a.nQB;
        w0 = (u % a.nQB) * 64;
        c0 = a.T_hist / 64 + u % a.nQB;
    }
    const int64_t b = bg / a.Hkv, g = bg % a.Hkv;

    __shared__ int s_ng;
    if (threadIdx.x == 0) {
        s_ng = 0;
        s_abort = 0;
        mbar_init(bar_q, 1);
        for (int rr = 0; rr < 2; ++rr)
            for (int s = 0; s < kStages; ++s) {
                mbar_init(bar_full(rr, s), 1);
                mbar_init(bar_empty(rr, s), 1);
            }
        for (int bb = 0; bb < 2; ++bb) {
            mbar_init(bar_s(bb), 1);
            mbar_init(bar_p(bb), kSoftmax);
            mbar_init(bar_o(bb), 1);
            for (int q = 0; q < 4; ++q) mbar_init(bar_mx(bb, q), 64);
        }
        mbar_init(bar_final, 1);
        mbar_init(bar_stage, kSoftmax);
        fence_mbar_init();
    }
    // Tensor memory: allocated here, or (ROUTED) once by the kernel for all its
    // tiles -- a CTA gives up its allocation permit after its first allocation.
    if constexpr (!ROUTED)
        if (warp == kMmaWarp) tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    // Setup above touches no global memory; the inputs are read from here on.
    pdl_wait();
    pdl_trigger();
    __syncthreads();
    wu::View uv{};
    if constexpr (CAUSAL) {
        // The union of the window's routed groups (eligible: before the own chunk).
        uv = wu::view(smem + L::union_off, a.n_groups, a.wg);
        wu::build(a.gidx + (bg * a.T_seg + w0) * a.wg, a.wg, 8 * c0, uv, &s_ng, chk::kSiteCausalFwd);
    } else {
        // Routed groups form a prefix of the row: count them with one parallel pass.
        int c = 0;
        for (int i = threadIdx.x; i < a.wg; i += kThreads) c += grow[i] >= 0;
        c = __reduce_add_sync(0xFFFFFFFFu, c);
        if (lane == 0 && c) atomicAdd(&s_ng, c);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_g = s_ng;
    const int n_rt = (n_g + 7) / 8;
    const int nt = n_rt + 1;                                // + own chunk tile
    // Column map: O at 0, S/P[b] at D + 64 b.
    constexpr uint32_t kColO = 0;
    auto col_s = [&](int bb) { return uint32_t(D + bb * kKeys); };

    const int64_t kv_base = bg * a.cap;                      // first K/V row of (b, g)

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer
        // Lane 0 issues the Q boxes and arms the barriers; for a routed tile,
        // lane j < 8 fetches group j's index and issues that group's boxes,
        // so the eight index loads overlap.
        if (lane == 0) {
            prefetch_tmap(tm_q);
            prefetch_tmap(tm_k8);
            prefetch_tmap(tm_v8);
            prefetch_tmap(tm_k64);
            prefetch_tmap(tm_v64);
            mbar_expect_tx(bar_q, 2 * H * 64 * 128);
            for (int hh = 0; hh < kHeads; ++hh) {
                const int head = head0 + hh;
                // A missing head (G not a multiple) is read past the end: zeros.
                const int y = head < a.G ? int((b * a.Hq + g * a.G + head) * a.T_seg + w0) : a.q_rows;
                for (int c = 0; c < H; ++c)
                    tma_load_2d(sbase + L::q_off + c * L::kQTile + hh * kRows * 128, tm_q, 64 * c, y, bar_q);
            }
        }
        // Lanes 0-7 load the K ring, lanes 8-15 the V ring, each at its own
        // pace: a K stage is free once S has read it, a V stage once PV has.
        if (lane < 16) {
            const int ring = lane / 8, gl = lane % 8, leader = 8 * ring;
            const unsigned mask = 0xFFu << (8 * ring);
            const CUtensorMap* m8 = ring == 0 ? tm_k8 : tm_v8;
            const CUtensorMap* m64 = ring == 0 ? tm_k64 : tm_v64;
            const uint32_t base = sbase + (ring == 0 ? L::k_off : L::v_off);
            for (int t = 0; t < nt; ++t) {
                const int s = t % kStages, r = t / kStages;
                bool ok = true;
                if (lane == leader) {
                    ok = t < kStages || mbar_wait(bar_empty(ring, s), (r - 1) & 1, kSiteEmpty);
                    if (ok) mbar_expect_tx(bar_full(ring, s), H * kKeys * 128);
                }
                if (!__shfl_sync(mask, ok, leader)) {
                    s_abort = 1;
                    break;
                }
                const uint32_t dst = base + s * H * L::kKVHalf;
                if (t < n_rt) {
                    const int gi = t * 8 + gl;
                    // Slots past the last routed group repeat group 0: finite
                    // data whose scores the softmax masks out.
                    int grp;
                    if constexpr (CAUSAL) grp = uv.list[gi < n_g ? gi : 0];   // checked when built
                    else if constexpr (ROUTED) grp = chk::group(grow[gi < n_g ? gi : 0], 8 * c0, chk::kSiteFwdTc);
                    else grp = chk::group(__ldg(grow + (gi < n_g ? gi : 0)), 8 * c0, chk::kSiteFwdTc);
                    const int y = int(kv_base + (int64_t)grp * 8);
                    for (int c = 0; c < H; ++c)
                        tma_load_2d(dst + c * L::kKVHalf + gl * 1024, m8, 64 * c, y, bar_full(ring, s));
                } else if (lane == leader) {
                    const int y = int(kv_base + 64 * c0);
                    for (int c = 0; c < H; ++c) tma_load_2d(dst + c * L::kKVHalf, m64, 64 * c, y, bar_full(ring, s));
                }
                __syncwarp(mask);
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(128, kKeys, 0, 0);
            constexpr uint32_t id_o = idesc_bf16(128, D, 0, 1);
            bool ok = mbar_wait(bar_q, 0, kSiteQ);
            // S runs two tiles ahead: S(t+2) overwrites the buffer of P(t) and
            // is issued right after PV(t) (MMAs of one thread run in order).
            auto issue_s = [&](int t) -> bool {
                const int s = t % kStages, bb = t & 1;
                if (!mbar_wait(bar_full(0, s), (t / kStages) & 1, kSiteFull)) return false;
                tc_fence_after();
                // Descriptors of the operand bases, stepped by constants.
                const uint64_t dq = sdesc_sw128(sbase + L::q_off, 16, 1024);
                const uint64_t dk = sdesc_sw128(sbase + L::k_off + s * H * L::kKVHalf, 16, 1024);
                const uint32_t ts = tmem + col_s(bb);
#pragma unroll
                for (int kk = 0; kk < 4 * H; ++kk)
                    mma_ss(ts, dq + (((kk / 4) * L::kQTile + (kk % 4) * 32) >> 4),
                           dk + (((kk / 4) * L::kKVHalf + (kk % 4) * 32) >> 4), id_s, kk > 0);
                mma_commit(bar_s(bb));
                mma_commit(bar_empty(0, s));                // K of this stage is read
                return true;
            };
            if (ok) ok = issue_s(0);
            if (ok && nt > 1) ok = issue_s(1);
            for (int t = 0; ok && t < nt; ++t) {
                const int s = t % kStages, bb = t & 1;
                if (!(ok = mbar_wait(bar_p(bb), (t / 2) & 1, kSiteP))) break;
                if (!(ok = mbar_wait(bar_full(1, s), (t / kStages) & 1, kSiteFull))) break;
                tc_fence_after();
                // P of keys 16kk.. : hi at column 16kk, lo at 16kk + 8.
                const uint64_t vd = sdesc_sw128(sbase + L::v_off + s * H * L::kKVHalf, L::kKVHalf, 1024);
                const uint32_t to = tmem + kColO, tp = tmem + col_s(bb);
                const bool acc = t > 0;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    mma_ts(to, tp + 16 * kk, vd + (kk * 16 * 128 >> 4), id_o, acc || kk > 0);
                    mma_ts(to, tp + 16 * kk + 8, vd + (kk * 16 * 128 >> 4), id_o, true);
                }
                mma_commit(bar_o(bb));
                mma_commit(bar_empty(1, s));                // V of this stage is read
                if (t + 2 < nt && !(ok = issue_s(t + 2))) break;
            }
            if (!ok) s_abort = 1;
            // Every MMA issued is complete before tensor memory is released.
            mma_commit(bar_final);
            mbar_wait(bar_final, 0, kSiteFinal);
        }
    } else {
        // ------------------------------------------------ softmax + epilogue
        // Thread (warp w, lane l): row r = 32(w%4) + l of the M-tile (its
        // tensor-memory lane) and keys 32 hk.. of each tile, hk = w/4.
        const int q = warp % 4, hk = warp / 4;
        const int r = 32 * q + lane;
        const int hp = r / kRows, pl = r % kRows;          // head within the tile, query within its rows
        const int i = int(w0) + pl;                        // query position within the segment
        const int own_lim = int(a.T_hist + i - 64 * c0);   // own-chunk keys 0 .. own_lim are visible
        const int head = head0 + hp;
        const uint32_t lane_off = uint32_t(32 * q) << 16;
        float m_run = -INFINITY;                           // same in both warps of the row
        float l_run = 0.f;                                 // over this thread's keys
        bool ok = true;
        for (int t = 0; t < nt && ok; ++t) {
            const int bb = t & 1;
            ok = mbar_wait(bar_s(bb), (t / 2) & 1, kSiteS);
            if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
            tc_fence_after();
            uint32_t raw[32];
            tmem_ld32(tmem + lane_off + col_s(bb) + 32 * hk, raw);
            tmem_wait_ld();
            float sv[32];
            const bool own = t == n_rt;
            // Full routed tiles need no masks (block path); the scale is applied
            // after the maximum (it is positive) and folded into the exponent's FMA.
            const bool full = !CAUSAL && !own && t * 8 + 8 <= n_g;
            // Causal: the masks of this warp's four group slots of the tile.
            uint32_t mb[4] = {0u, 0u, 0u, 0u};
            if constexpr (CAUSAL) {
                if (!own) {
#pragma unroll
                    for (int s4 = 0; s4 < 4; ++s4) {
                        const int slot = t * 8 + 4 * hk + s4;
                        mb[s4] = slot < n_g ? uv.mask[slot] : 0u;
                    }
                }
            }
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int jj = 32 * hk + j;                // key within the tile
                sv[j] = __uint_as_float(raw[j]);
                if constexpr (CAUSAL) {
                    bool vis;
                    if (own) vis = jj <= own_lim;
                    else vis = (mb[j / 8] >> pl) & 1u;
                    if (!vis) sv[j] = -INFINITY;
                } else {
                    // One expression: written through the causal variant's
                    // `vis` the block path's tile loop measured 45 against 39 us
                    // at 16K (the compiler schedules it differently).
                    if (!full && !(own ? (jj <= pl) : (t * 8 + jj / 8 < n_g))) sv[j] = -INFINITY;
                }
                m4[j & 3] = fmaxf(m4[j & 3], sv[j]);
            }
            const float pm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * a.scale_log2;
            // The row's maximum over the tile: exchange with the other warp of
            // the quadrant (bounded wait; both then take the same decisions).
            float* xs = xmax + (bb * 4 + q) * 64;
            xs[32 * hk + lane] = pm;
            mbar_arrive(bar_mx(bb, q));
            ok = mbar_wait(bar_mx(bb, q), (t / 2) & 1, kSiteMax);
            if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
            const float mx = fmaxf(pm, xs[32 * (1 - hk) + lane]);
            const bool need = mx > m_run + kRescaleLog2;
            if (__any_sync(0xFFFFFFFFu, need)) {
                const float m_new = need ? mx : m_run;
                // 0 when m_run = -inf; 1 for a lane that keeps its maximum (also
                // one that has seen no visible key yet: -inf - -inf is no number).
                const float alpha = CAUSAL ? (need ? fast_exp2(m_run - m_new) : 1.f) : fast_exp2(m_run - m_new);
                if (t > 0) {
                    ok = mbar_wait(bar_o((t - 1) & 1), ((t - 1) / 2) & 1, kSiteO);
                    if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
                    tc_fence_after();
                    // This warp's half of O's columns.
#pragma unroll 1
                    for (int c = 0; c < D / 64; ++c) {
                        const uint32_t col = kColO + (D / 2) * hk + 32 * c;
                        uint32_t ov[32];
                        tmem_ld32(tmem + lane_off + col, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
                        tmem_st32(tmem + lane_off + col, ov);
                    }
                    tmem_wait_st();
                }
                l_run *= alpha;
                m_run = m_new;
            }
            // P = hi + lo, both bf16: the two MMAs carry P to ~14 bits, where
            // one bf16 operand alone (8 bits) misses the 2e-3 output bound.
            // Keys 16kk.. of the tile: hi at column 16kk, lo at 16kk + 8, so
            // the warp writes only the 32 columns it read.
            uint32_t pk[32];
            float2 rs = make_float2(0.f, 0.f);
            // No visible key yet (a causal row whose position routed none of the
            // tiles so far): every score is -inf, and subtracting 0 keeps
            // exp2(-inf) = 0 rather than -inf + inf.
            const float mz = CAUSAL ? (m_run == -INFINITY ? 0.f : -m_run) : -m_run;
            const float2 c2 = make_float2(a.scale_log2, a.scale_log2), nm = make_float2(mz, mz);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float2 x = __ffma2_rn(make_float2(sv[2 * j], sv[2 * j + 1]), c2, nm);
                const float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                rs = __fadd2_rn(rs, p);
                split_bf16x2(p.x, p.y, pk[16 * (j / 8) + j % 8], pk[16 * (j / 8) + 8 + j % 8]);
            }
            l_run += rs.x + rs.y;
            tmem_st32(tmem + lane_off + col_s(bb) + 32 * hk, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p(bb));
        }
        if (ok) {
            ok = mbar_wait(bar_o((nt - 1) & 1), ((nt - 1) / 2) & 1, kSiteO);
            if (__any_sync(0xFFFFFFFFu, !ok)) ok = false;
        }
        float l_row = 0.f;
        if (ok) {
            // The row sum: both warps' partial sums, through the exchange slot
            // of tile nt (its last use, tile nt - 2, is read by both).
            const int bx = nt & 1;
            float* xs = xmax + (bx * 4 + q) * 64;
            xs[32 * hk + lane] = l_run;
            mbar_arrive(bar_mx(bx, q));
            ok = mbar_wait(bar_mx(bx, q), (nt / 2) & 1, kSiteMax);
            if (__any_sync(0xFFFFFFFFu, !ok)) ok = false;
            l_row = l_run + xs[32 * (1 - hk) + lane];
        }
        if (ok) {
            // O = acc / l through a swizzled shared-memory stage (the Q and
            // K/V buffers are free once the last PV is done), then coalesced
            // row stores.  Each warp stages its half of the row's columns.
            tc_fence_after();
            float* stage = reinterpret_cast<float*>(smem + L::q_off);
            const float inv = 1.f / l_row;
#pragma unroll 1
            for (int c = 0; c < D / 64; ++c) {
                const int c32 = (D / 64) * hk + c;          // 32-column chunk of the row
                uint32_t ov[32];
                tmem_ld32(tmem + lane_off + kColO + 32 * c32, ov);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const int ch = (32 * c32 + j) / 4;
                    const int pch = (ch & ~7) | ((ch ^ r) & 7);
                    *reinterpret_cast<float4*>(stage + r * D + 4 * pch) =
                        make_float4(__uint_as_float(ov[j]) * inv, __uint_as_float(ov[j + 1]) * inv,
                                    __uint_as_float(ov[j + 2]) * inv, __uint_as_float(ov[j + 3]) * inv);
                }
            }
            if (hk == 0 && head < a.G) {
                const int64_t row = ((b * a.Hq + g * a.G + head) * a.T_seg + i);
                a.lse[row] = (m_run + log2f(l_row)) * kLn2;
            }
            // All softmax threads have staged their rows (bounded wait).
            mbar_arrive(bar_stage);
            if (!mbar_wait(bar_stage, 0, kSiteStage)) s_abort = 1;
            constexpr int C4 = D / 4;                      // 16-byte chunks per row
            for (int rr = warp; rr < 128; rr += kSoftmaxWarps) {
                const int head_r = head0 + rr / kRows;
                if (head_r >= a.G) continue;
                const int64_t grow_ = (b * a.Hq + g * a.G + head_r) * a.T_seg + w0 + rr % kRows;
                for (int ch = lane; ch < C4; ch += 32) {
                    const int pch = (ch & ~7) | ((ch ^ rr) & 7);
                    *reinterpret_cast<float4*>(a.O + grow_ * D + 4 * ch) =
                        *reinterpret_cast<const float4*>(stage + rr * D + 4 * pch);
                }
            }
        } else {
            s_abort = 1;
        }
    }

    // ---- wind down: every TMA copy this CTA issued has landed before exit
    tc_fence_before();
    __syncthreads();
    if (s_abort && warp == kProducerWarp && lane == 0) {
        for (int rr = 0; rr < 2; ++rr)
            for (int s = 0; s < kStages; ++s) {
                // Loads issued for stage s: tiles s, s+S, ... < nt; wait for the last.
                int last = -1;
                for (int t = s; t < nt; t += kStages) last = t;
                if (last >= 0) mbar_wait(bar_full(rr, s), (last / kStages) & 1, kSiteDrain);
            }
        mbar_wait(bar_q, 0, kSiteDrain);
    }
    __syncthreads();
    if constexpr (!ROUTED) {
        if (warp == kMmaWarp) {
            tc_fence_after();
            tmem_dealloc(tmem, L::kTmemCols);
        }
    }
}

// CTAs of one query block are adjacent, so they run together and share the
// K/V tiles through L2.  Strictly causal variant: CTA x runs window item
// sched[x], the items ordered heaviest first (one item per CTA, and an
// item's time grows with its union's key tiles).
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 2)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k8,
                   const __grid_constant__ CUtensorMap tm_v8, const __grid_constant__ CUtensorMap tm_k64,
                   const __grid_constant__ CUtensorMap tm_v64, const FwdArgs a)
{
    constexpr int kHeads = CAUSAL ? 4 : 2;
    const int n_y = (a.G + kHeads - 1) / kHeads;
    int64_t it = blockIdx.x;
    if constexpr (CAUSAL) {
        // The items' order is an input: read once the previous launch is done.
        pdl_wait();
        it = chk::sched_item(a.sched);
    }
    const int64_t u = it / n_y;                             // ((b*Hkv)+g)*nQB + qb, or the window
    fwd_tile<D, CAUSAL, false>(&tm_q, &tm_k8, &tm_v8, &tm_k64, &tm_v64, a, u, kHeads * int(it % n_y),
                               a.gidx + u * a.wg);
}

// ---- routing and forward in one persistent launch ---------------------------------------------------
struct RouteArgs {
    const __nv_bfloat16* Q;
    const float* csum;
    const float* gsum;
    float* qbar;
    int32_t* cidx;
    int32_t* gidx;
    int64_t n_blocks, nC, nCs, nGs, c_hist;
    int k_c, wc, k_g;
    float inv_rows;
};

// Routing scratch of the fused kernel, inside the K / V rings (free until a
// tile's loads start): the router's row partial sums, the block query, the
// candidate keys, ids, chosen chunks and flags.
template <int D>
struct RouteScratch {
    static constexpr int RL = rt::kRouterThreads / (D / 8);   // row lanes of the block query (bf16)
    static constexpr int part_off = 0;
    static constexpr int qs_off = part_off + RL * D * 4;
    static constexpr int keys_off = qs_off + D * 4;
    __host__ __device__ static size_t bytes(int64_t nC, int wc)
    {
        const size_t nk = (size_t)(nC > 8 * (int64_t)wc ? nC : 8 * (int64_t)wc);
        return keys_off + 8 * nk + 4 * 8 * (size_t)wc + 4 * (size_t)wc + 8 * (size_t)wc;
    }
};

// CTA x takes query blocks x, x + gridDim.x, ...: for each, warps 0-7 run the
// router's a2-a4 pieces for the block (block query, chunk and group
// routing; qbar, cidx, gidx written as hga_route writes them) and keep its
// group row in shared memory, then the CTA runs the forward tile of every
// q-head pair of the block on that row.  One launch replaces the router's
// and the forward's; the block's K / V tiles are read by its head pairs one
// after another from L2.  (Routing the block again in every head pair's
// tile, so that the pairs run on different CTAs at once, measured slower:
// 61 against 52 us at 16K.)
template <int D>
__global__ void __launch_bounds__(kThreads, 2)
route_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k8,
                      const __grid_constant__ CUtensorMap tm_v8, const __grid_constant__ CUtensorMap tm_k64,
                      const __grid_constant__ CUtensorMap tm_v64, const FwdArgs a, const RouteArgs r)
{
    using L = FwdSmem<D>;
    using RS = RouteScratch<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* scratch = smem + L::k_off;
    float(*part)[D] = reinterpret_cast<float(*)[D]>(scratch + RS::part_off);
    float* qs = reinterpret_cast<float*>(scratch + RS::qs_off);
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(scratch + RS::keys_off);
    const size_t nk = (size_t)(r.nC > 8 * (int64_t)r.wc ? r.nC : 8 * (int64_t)r.wc);
    int32_t* ids = reinterpret_cast<int32_t*>(keys + nk);
    int32_t* crow = ids + 8 * r.wc;
    uint8_t* flags = reinterpret_cast<uint8_t*>(crow + r.wc);
    int32_t* grow = reinterpret_cast<int32_t*>(smem + L::union_off);   // the block's group row
    __shared__ int s_nvalid;
    const int warp = threadIdx.x / 32;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::tmem_slot_off);
    if (warp == kMmaWarp) tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);   // for every tile of the CTA
    pdl_wait();
    pdl_trigger();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int n_y = (a.G + 1) / 2;
    for (int64_t u = blockIdx.x; u < r.n_blocks; u += gridDim.x) {
        const int64_t qb = u % a.nQB, bg = u / a.nQB;
        const int64_t b = bg / a.Hkv, g = bg % a.Hkv;
        if (threadIdx.x < rt::kRouterThreads) {
            const int tid = threadIdx.x;
            rt::block_query<__nv_bfloat16, D, rt::SyncRouterThreads>(r.Q, r.qbar + u * D, qs, part, b, g, qb, a.Hq,
                                                                      a.G, a.T_seg, r.inv_rows, tid);
            rt::route_chunks_block<D, rt::SyncRouterThreads>(qs, r.csum + bg * r.nCs * D, int(r.c_hist + qb), r.k_c,
                                                             r.wc, keys, r.cidx + u * r.wc, crow, tid);
            rt::route_groups_block<D, rt::SyncRouterThreads>(qs, r.gsum + bg * r.nGs * D, crow, r.wc, r.k_g, a.wg,
                                                             keys, ids, flags, &s_nvalid, grow, tid);
        }
        __syncthreads();                                    // the group row is complete
        for (int i = threadIdx.x; i < a.wg; i += kThreads) r.gidx[u * a.wg + i] = grow[i];
        for (int hp = 0; hp < n_y; ++hp)
            fwd_tile<D, false, true>(&tm_q, &tm_k8, &tm_v8, &tm_k64, &tm_v64, a, u, 2 * hp, grow);
    }
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(*tmem_slot, L::kTmemCols);
    }
}

// ---- host side -------------------------------------------------------------------------------------
template <int D, bool CAUSAL>
cudaError_t launch(const Shape& s, const void* Q, const void* K, const void* V, const int32_t* gidx,
                   const int32_t* sched, float* O, float* lse, cudaStream_t st)
{
    CUtensorMap tq, tk8, tv8, tk64, tv64;
    constexpr int kRows = CAUSAL ? wu::kWin : 64;           // query rows of a head in a tile
    const uint64_t q_rows = (uint64_t)s.B * s.Hq * s.T_seg, kv_rows = (uint64_t)s.B * s.Hkv * s.cap;
    if (!make_bf16_map(&tq, Q, q_rows, D, kRows) || !make_bf16_map(&tk8, K, kv_rows, D, 8) ||
        !make_bf16_map(&tv8, V, kv_rows, D, 8) || !make_bf16_map(&tk64, K, kv_rows, D, 64) ||
        !make_bf16_map(&tv64, V, kv_rows, D, 64))
        return cudaErrorInvalidValue;
    FwdArgs a;
    a.gidx = gidx;
    a.O = O;
    a.lse = lse;
    a.Hq = s.Hq;
    a.Hkv = s.Hkv;
    a.G = s.G;
    a.wg = s.wg;
    a.T_hist = s.T_hist;
    a.T_seg = s.T_seg;
    a.nQB = s.nQB;
    a.q_rows = (int)q_rows;
    a.kv_rows = (int)kv_rows;
    a.cap = s.cap;
    a.scale_log2 = s.scale * kLog2e;
    a.nWin = s.T_seg / wu::kWin;
    a.n_groups = s.nG;
    a.sched = CAUSAL ? sched : nullptr;
    // One tile (a head pair of a query block, or four heads of a causal
    // window) per CTA, two CTAs per SM when shared memory allows.
    auto k = attn_fwd_tc_kernel<D, CAUSAL>;
    const int smem = CAUSAL ? int(FwdSmem<D>::union_off + wu::bytes(s.nG, s.wg) + 1024) : FwdSmem<D>::alloc;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int64_t ctas = CAUSAL ? (int64_t)s.B * s.Hkv * a.nWin * ((s.G + 3) / 4)
                                : (int64_t)s.B * s.Hkv * s.nQB * ((s.G + 1) / 2);
    return launch_pdl(k, dim3((unsigned)ctas), dim3(kThreads), (size_t)smem, st, tq, tk8, tv8, tk64, tv64, a);
}

template <int D>
cudaError_t launch_route_fwd(const Shape& s, const void* Q, const void* K, const void* V, const float* csum,
                             const float* gsum, float* qbar, int32_t* cidx, int32_t* gidx, float* O, float* lse,
                             cudaStream_t st)
{
    CUtensorMap tq, tk8, tv8, tk64, tv64;
    const uint64_t q_rows = (uint64_t)s.B * s.Hq * s.T_seg, kv_rows = (uint64_t)s.B * s.Hkv * s.cap;
    if (!make_bf16_map(&tq, Q, q_rows, D, 64) || !make_bf16_map(&tk8, K, kv_rows, D, 8) ||
        !make_bf16_map(&tv8, V, kv_rows, D, 8) || !make_bf16_map(&tk64, K, kv_rows, D, 64) ||
        !make_bf16_map(&tv64, V, kv_rows, D, 64))
        return cudaErrorInvalidValue;
    FwdArgs a{};
    a.gidx = gidx;
    a.O = O;
    a.lse = lse;
    a.Hq = s.Hq;
    a.Hkv = s.Hkv;
    a.G = s.G;
    a.wg = s.wg;
    a.T_hist = s.T_hist;
    a.T_seg = s.T_seg;
    a.nQB = s.nQB;
    a.q_rows = (int)q_rows;
    a.kv_rows = (int)kv_rows;
    a.cap = s.cap;
    a.scale_log2 = s.scale * kLog2e;
    RouteArgs r{};
    r.Q = static_cast<const __nv_bfloat16*>(Q);
    r.csum = csum;
    r.gsum = gsum;
    r.qbar = qbar;
    r.cidx = cidx;
    r.gidx = gidx;
    r.n_blocks = (int64_t)s.B * s.Hkv * s.nQB;
    r.nC = s.nC;
    r.nCs = s.nCs;
    r.nGs = s.nGs;
    r.c_hist = s.T_hist / kChunk;
    r.k_c = s.k_c;
    r.wc = s.wc;
    r.k_g = s.k_g;
    r.inv_rows = 1.0f / (float)(s.G * kChunk);
    auto k = route_attn_fwd_kernel<D>;
    const int smem = int(FwdSmem<D>::union_off + 4 * (size_t)s.wg + 1024);
    cudaError_t e = allow_smem(k, smem);
    if (e != cudaSuccess) return e;
    // Two CTAs per SM, each walking query blocks.
    const int64_t grid = std::min<int64_t>(r.n_blocks, 2 * (int64_t)sm_count());
    return launch_pdl(k, dim3((unsigned)grid), dim3(kThreads), (size_t)smem, st, tq, tk8, tv8, tk64, tv64, a, r);
}

}  // namespace

int attn_fwd_tc_status(bool clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, sm100::g_status, sizeof v) != cudaSuccess) return -1;
    if (clear && v) {
        const int z = 0;
        cudaMemcpyToSymbol(sm100::g_status, &z, sizeof z);
    }
    return v;
}

bool attn_fwd_tc_supported(const Shape& s)
{
    const uint64_t q_rows = (uint64_t)s.B * s.Hq * s.T_seg, kv_rows = (uint64_t)s.B * s.Hkv * s.cap;
    return s.dtype == HGA_BF16 && (s.d == 128 || s.d == 64) && q_rows < (1ull << 31) &&
           kv_rows < (1ull << 31) && tensor_maps_available();
}

cudaError_t launch_attn_fwd_tc(const Shape& s, const void* Q, const void* K, const void* V,
                               const int32_t* gidx, float* O, float* lse, cudaStream_t st)
{
    return s.d == 128 ? launch<128, false>(s, Q, K, V, gidx, nullptr, O, lse, st)
                      : launch<64, false>(s, Q, K, V, gidx, nullptr, O, lse, st);
}

// Routing and forward in one launch: the tensor-core forward's shapes whose
// routing scratch fits in the K / V rings and whose group row fits beside
// the forward's shared memory.
bool route_attn_fwd_tc_supported(const Shape& s)
{
    if (!attn_fwd_tc_supported(s)) return false;
    const size_t rings = s.d == 128 ? FwdSmem<128>::xmax_off - FwdSmem<128>::k_off
                                    : FwdSmem<64>::xmax_off - FwdSmem<64>::k_off;
    const size_t scratch = s.d == 128 ? RouteScratch<128>::bytes(s.nC, s.wc) : RouteScratch<64>::bytes(s.nC, s.wc);
    const size_t smem = (size_t)(s.d == 128 ? FwdSmem<128>::union_off : FwdSmem<64>::union_off) + 4 * (size_t)s.wg +
                        1024;
    return scratch <= rings && smem <= 227 * 1024 / 2;
}

cudaError_t launch_route_attn_fwd_tc(const Shape& s, const void* Q, const void* K, const void* V, const float* csum,
                                     const float* gsum, float* qbar, int32_t* cidx, int32_t* gidx, float* O,
                                     float* lse, cudaStream_t st)
{
    return s.d == 128 ? launch_route_fwd<128>(s, Q, K, V, csum, gsum, qbar, cidx, gidx, O, lse, st)
                      : launch_route_fwd<64>(s, Q, K, V, csum, gsum, qbar, cidx, gidx, O, lse, st);
}

// Strictly causal variant on the tensor cores: bf16, index rows of at most
// 64 groups (a window's union of at most 2048), shared memory permitting.
bool attn_fwd_tc_causal_supported(const Shape& s)
{
    const size_t smem = (size_t)(s.d == 128 ? FwdSmem<128>::union_off : FwdSmem<64>::union_off) +
                        wu::bytes(s.nG, s.wg) + 1024;
    return attn_fwd_tc_supported(s) && s.wg <= 64 && s.T_seg % wu::kWin == 0 && smem <= 227 * 1024;
}

cudaError_t launch_attn_fwd_tc_causal(const Shape& s, const void* Q, const void* K, const void* V,
                                      const int32_t* gidx, const int32_t* sched, float* O, float* lse,
                                      cudaStream_t st)
{
    return s.d == 128 ? launch<128, true>(s, Q, K, V, gidx, sched, O, lse, st)
                      : launch<64, true>(s, Q, K, V, gidx, sched, O, lse, st);
}

// Check word of this translation unit's bounds checks (checked builds).
HGA_CHECK_WORD_READER(check_word_attn_tc_fwd)

}  // namespace hga
