// attn_tc_bwd.cu -- a6 routed attention backward on the tcgen05 tensor cores
// (bf16 inputs, d = 128, float32 accumulation).
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
//     P   = exp2(S*c - lse), dS = P (dP - D)   row per thread; both written
//           to shared memory as bf16 hi + lo parts (~14-bit operands)
//     dQ += dS K                      A = dS (K-major), B = K (MN-major)
//     dV^T = dO^T P, dK^T = Q^T dS    A = dO / Q read MN-major, B = P / dS
// dV^T and dK^T (d on the tensor-memory lanes, keys on the columns) are added
// to the float32 dV_seg / dK_seg rows of the segment's keys with coalesced
// atomics; tiles whose keys are all detached history skip both products
// (routed groups are ascending, so history tiles come first).
//
// Warp roles (576 threads): warps 0-15 compute P and dS (row 32*(w%4)+lane,
// 16-key quarter w/4; four warps per scheduler hide each other's latency),
// add the previous tile's dK/dV while the MMAs of the current one run, and
// write dQ at the end; warp 16 is the TMA producer, warp 17 the
// tensor-memory owner and MMA issuer.  Tensor memory (512 columns): S and dP
// double-buffered (4 x 64), dQ (128), dV^T (64), dK^T (64).  Three K/V
// stages (224 KB of shared memory in all) keep the gathered loads two tiles
// ahead of the MMAs.
#include <algorithm>

#include "hga_internal.cuh"
#include "sm100.cuh"

namespace hga {
namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int H = 2;                  // 64-column halves of d
constexpr int kStages = 3;
constexpr int kKeys = 64;
constexpr int kComputeWarps = 16;     // 4 per lane quadrant, one 16-key quarter each
constexpr int kCompute = 32 * kComputeWarps;
constexpr int kProducerWarp = kComputeWarps, kMmaWarp = kComputeWarps + 1;
constexpr int kThreads = 32 * (kComputeWarps + 2);
constexpr float kLog2e = 1.4426950408889634f;

enum : int {
    kSiteQ = 201, kSiteFull, kSiteEmpty, kSiteSdp, kSitePs, kSiteMm2, kSiteDrained, kSiteFinal, kSiteDrain,
    kSiteQfree, kSiteDqfree, kSiteStage
};

struct BwdSmem {
    static constexpr int kRows128 = 128 * 128;        // 128 rows x 128 B
    static constexpr int kKVHalf = kKeys * 128;       // 64 keys x 128 B
    static constexpr int q_off = 0;                   // [2 halves][128 rows][64]
    static constexpr int do_off = q_off + H * kRows128;
    static constexpr int k_off = do_off + H * kRows128;
    static constexpr int v_off = k_off + kStages * H * kKVHalf;
    static constexpr int p_off = v_off + kStages * H * kKVHalf;   // P hi, P lo: [128 rows][64 keys]
    static constexpr int ds_off = p_off + 2 * kRows128;           // dS hi, dS lo
    static constexpr int bar_off = ds_off + 2 * kRows128;
    // q, full[S], empty[S], sdp[2], ps, mm2, drained, final, qfree, dqfree, stage
    static constexpr int n_bars = 1 + 2 * kStages + 2 + 7;
    static constexpr int tmem_slot_off = bar_off + 8 * n_bars;
    static constexpr int bytes = tmem_slot_off + 16;
    static constexpr int alloc = bytes + 1024;
};

// Tensor-memory columns.
constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256, kColDV = 384, kColDK = 448;

struct BwdArgs {
    const int32_t* gidx;
    const float* lse;
    const float* Drow;
    float* dQ;
    float* dK;
    float* dV;
    int Hq, Hkv, G, wg;
    int64_t T_hist, T_seg, nQB, n_items;
    int q_rows;
    float scale, scale_log2;
};

// Does key tile t hold any segment token (position >= T_hist)?
__device__ __forceinline__ bool tile_has_segment_keys(int t, int n_rt, int n_g, const int32_t* grow,
                                                      int64_t T_hist)
{
    if (t == n_rt) return true;                              // own chunk
    const int last = min(t * 8 + 7, n_g - 1);
    return (int64_t)grow[last] * 8 + 7 >= T_hist;
}

// One work item: a (batch, kv-head, query block) and a pair of its q-heads.
struct Item {
    int64_t bg, qb, b, g, kv_base, own_start, u;
    int head0, n_g, n_rt, nt;
    uint64_t seg;                   // bit t: key tile t holds segment tokens (t < 64)
    const int32_t* grow;
};

// Decode item `it` and count its routed groups (an ascending prefix of the
// index row).  Whole-warp call.
__device__ __forceinline__ Item make_item(const BwdArgs& a, int64_t it, int lane)
{
    Item m;
    const int n_pairs = (a.G + 1) / 2;
    m.u = it / n_pairs;                                     // (b*Hkv + g)*nQB + qb
    m.head0 = 2 * int(it % n_pairs);
    m.qb = m.u % a.nQB;
    m.bg = m.u / a.nQB;
    m.b = m.bg / a.Hkv;
    m.g = m.bg % a.Hkv;
    m.kv_base = m.bg * (a.T_hist + a.T_seg);
    m.own_start = a.T_hist + m.qb * 64;
    m.grow = a.gidx + m.u * a.wg;
    // Count the routed groups and mark the tiles holding segment groups
    // (group j is a segment group when 8 j >= T_hist).
    int c = 0;
    uint64_t seg = 0;
    const int64_t first_seg_group = a.T_hist / 8;
    for (int base = 0; base < a.wg; base += 32) {
        const int i = base + lane;
        const int32_t j = i < a.wg ? __ldg(m.grow + i) : -1;
        c += j >= 0;
        const unsigned in_seg = __ballot_sync(0xFFFFFFFFu, j >= 0 && j >= first_seg_group);
        for (int q = 0; q < 4 && base / 8 + q < 64; ++q)
            if ((in_seg >> (8 * q)) & 0xFFu) seg |= 1ull << (base / 8 + q);
    }
    m.n_g = __reduce_add_sync(0xFFFFFFFFu, c);
    m.n_rt = (m.n_g + 7) / 8;
    m.nt = m.n_rt + 1;
    if (m.n_rt < 64) seg |= 1ull << m.n_rt;                 // the own chunk
    m.seg = seg;
    return m;
}

// Does key tile t of item m hold any segment token (position >= T_hist)?
__device__ __forceinline__ bool item_tile_has_segment_keys(const Item& m, int t, int64_t T_hist)
{
    if (t < 64) return (m.seg >> t) & 1ull;
    return tile_has_segment_keys(t, m.n_rt, m.n_g, m.grow, T_hist);
}

// Persistent: CTA c processes items c, c + gridDim.x, ...  Barrier phases
// run on a global key-tile counter (gt) and an item counter (k) that every
// role advances identically, so the next item's loads and first S/dP MMAs
// overlap the current item's dK/dV and dQ epilogues.
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_k8, const __grid_constant__ CUtensorMap tm_v8,
                   const __grid_constant__ CUtensorMap tm_k64, const __grid_constant__ CUtensorMap tm_v64,
                   const BwdArgs a)
{
    using L = BwdSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::bar_off;
    const uint32_t bar_q = bar0;
    auto bar_full = [&](int s) { return bar0 + 8 * (1 + s); };
    auto bar_empty = [&](int s) { return bar0 + 8 * (1 + kStages + s); };
    auto bar_sdp = [&](int b) { return bar0 + 8 * (1 + 2 * kStages + b); };
    const uint32_t bar_ps = bar0 + 8 * (3 + 2 * kStages);
    const uint32_t bar_mm2 = bar0 + 8 * (4 + 2 * kStages);
    const uint32_t bar_drained = bar0 + 8 * (5 + 2 * kStages);
    const uint32_t bar_final = bar0 + 8 * (6 + 2 * kStages);
    const uint32_t bar_qfree = bar0 + 8 * (7 + 2 * kStages);
    const uint32_t bar_dqfree = bar0 + 8 * (8 + 2 * kStages);
    const uint32_t bar_stage = bar0 + 8 * (9 + 2 * kStages);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::tmem_slot_off);
    __shared__ int s_abort;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t n_items = a.n_items;

    if (threadIdx.x == 0) {
        s_abort = 0;
        mbar_init(bar_q, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        mbar_init(bar_sdp(0), 1);
        mbar_init(bar_sdp(1), 1);
        mbar_init(bar_ps, kCompute);
        mbar_init(bar_mm2, 1);
        mbar_init(bar_drained, kCompute);
        mbar_init(bar_final, 1);
        mbar_init(bar_qfree, 1);
        mbar_init(bar_dqfree, kCompute);
        mbar_init(bar_stage, kCompute);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) tmem_alloc(smem_u32(tmem_slot), 512);
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
        int last_gt[kStages] = {-1, -1, -1};                // last tile loaded per stage
        int k_loaded = -1;                                  // last item whose Q/dO was loaded
        uint32_t gt = 0;
        bool ok = true;
        int k = 0;
        for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++k) {
            const Item m = make_item(a, it, lane);
            for (int t = 0; t < m.nt && ok; ++t, ++gt) {
                const int s = gt % kStages;
                if (lane == 0) {
                    ok = gt < kStages || mbar_wait(bar_empty(s), ((gt / kStages) - 1) & 1, kSiteEmpty);
                    if (ok) mbar_expect_tx(bar_full(s), 2 * H * kKeys * 128);
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) break;
                last_gt[s] = gt;
                const uint32_t kdst = sbase + L::k_off + s * H * L::kKVHalf;
                const uint32_t vdst = sbase + L::v_off + s * H * L::kKVHalf;
                if (t < m.n_rt) {
                    if (lane < 8) {                           // one group per lane
                        const int gi = t * 8 + lane;
                        const int grp = __ldg(m.grow + (gi < m.n_g ? gi : 0));
                        const int y = int(m.kv_base + (int64_t)grp * 8);
                        for (int c = 0; c < H; ++c) {
                            tma_load_2d(kdst + c * L::kKVHalf + lane * 1024, &tm_k8, 64 * c, y, bar_full(s));
                            tma_load_2d(vdst + c * L::kKVHalf + lane * 1024, &tm_v8, 64 * c, y, bar_full(s));
                        }
                    }
                } else if (lane == 0) {
                    const int y = int(m.kv_base + m.own_start);
                    for (int c = 0; c < H; ++c) {
                        tma_load_2d(kdst + c * L::kKVHalf, &tm_k64, 64 * c, y, bar_full(s));
                        tma_load_2d(vdst + c * L::kKVHalf, &tm_v64, 64 * c, y, bar_full(s));
                    }
                }
                __syncwarp();
                if (t == 0) {
                    // Q and dO of this item once the previous item's MMAs are done.
                    if (lane == 0) {
                        ok = k == 0 || mbar_wait(bar_qfree, (k - 1) & 1, kSiteQfree);
                        if (ok) {
                            mbar_expect_tx(bar_q, 2 * 2 * H * 64 * 128);
                            for (int hp = 0; hp < 2; ++hp) {
                                const int head = m.head0 + hp;
                                const int y = head < a.G
                                                  ? int((m.b * a.Hq + m.g * a.G + head) * a.T_seg + m.qb * 64)
                                                  : a.q_rows;
                                for (int c = 0; c < H; ++c) {
                                    const uint32_t off = c * L::kRows128 + hp * 64 * 128;
                                    tma_load_2d(sbase + L::q_off + off, &tm_q, 64 * c, y, bar_q);
                                    tma_load_2d(sbase + L::do_off + off, &tm_do, 64 * c, y, bar_q);
                                }
                            }
                        }
                    }
                    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                    if (ok) k_loaded = k;
                }
            }
        }
        if (!ok) s_abort = 1;
        // Wind down: every copy issued has landed before the CTA exits.
        __syncwarp();
        if (lane == 0 && !ok) {
            for (int s = 0; s < kStages; ++s)
                if (last_gt[s] >= 0) mbar_wait(bar_full(s), (last_gt[s] / kStages) & 1, kSiteDrain);
            if (k_loaded >= 0) mbar_wait(bar_q, k_loaded & 1, kSiteDrain);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        constexpr uint32_t id_sdp = idesc_bf16(128, kKeys, 0, 0);   // S, dP
        constexpr uint32_t id_dq = idesc_bf16(128, D, 0, 1);        // dQ: A dS K-major, B K MN-major
        constexpr uint32_t id_kv = idesc_bf16(128, kKeys, 1, 1);    // dV^T, dK^T: both MN-major
        uint32_t gt = 0;
        bool ok = true;
        int k = 0;
        for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++k) {
            const Item m = make_item(a, it, lane);
            if (lane == 0) {
                auto issue_sdp = [&](uint32_t gtt) -> bool {
                    const int s = gtt % kStages, bb = gtt & 1;
                    if (!mbar_wait(bar_full(s), (gtt / kStages) & 1, kSiteFull)) return false;
                    tc_fence_after();
                    for (int kk = 0; kk < 4 * H; ++kk) {
                        const uint32_t o = (kk / 4) * L::kRows128 + (kk % 4) * 32;
                        const uint32_t ko = (s * H + kk / 4) * L::kKVHalf + (kk % 4) * 32;
                        mma_ss(tmem + kColS + bb * kKeys, sdesc_sw128(sbase + L::q_off + o, 16, 1024),
                               sdesc_sw128(sbase + L::k_off + ko, 16, 1024), id_sdp, kk > 0);
                        mma_ss(tmem + kColDP + bb * kKeys, sdesc_sw128(sbase + L::do_off + o, 16, 1024),
                               sdesc_sw128(sbase + L::v_off + ko, 16, 1024), id_sdp, kk > 0);
                    }
                    mma_commit(bar_sdp(bb));
                    return true;
                };
                ok = mbar_wait(bar_q, k & 1, kSiteQ);
                // S / dP run two tiles ahead (double-buffered): S(t+2) is
                // issued right after the MMAs of tile t, so its load wait never
                // holds back the gradient MMAs of the tile the softmax finished.
                if (ok) ok = issue_sdp(gt);
                if (ok && m.nt > 1) ok = issue_sdp(gt + 1);
                for (int t = 0; ok && t < m.nt; ++t) {
                    const uint32_t gtt = gt + t;
                    const int s = gtt % kStages;
                    if (!(ok = mbar_wait(bar_ps, gtt & 1, kSitePs))) break;
                    // dQ accumulates from zero: the previous item's dQ is read out.
                    if (t == 0 && k > 0 && !(ok = mbar_wait(bar_dqfree, (k - 1) & 1, kSiteDqfree))) break;
                    tc_fence_after();
                    // dQ += dS K  (dS hi and lo against the same K)
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t kb =
                            sdesc_sw128(sbase + L::k_off + s * H * L::kKVHalf + kk * 2048, L::kKVHalf, 1024);
                        mma_ss(tmem + kColDQ, sdesc_sw128(sbase + L::ds_off + kk * 32, 16, 1024), kb, id_dq,
                               t > 0 || kk > 0);
                        mma_ss(tmem + kColDQ, sdesc_sw128(sbase + L::ds_off + L::kRows128 + kk * 32, 16, 1024), kb,
                               id_dq, true);
                    }
                    if (item_tile_has_segment_keys(m, t, a.T_hist)) {
                        if (gtt >= 1 && !(ok = mbar_wait(bar_drained, (gtt - 1) & 1, kSiteDrained))) break;
                        tc_fence_after();
                        // dV^T = dO^T P and dK^T = Q^T dS over the 128 query rows.
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t dOt = sdesc_sw128(sbase + L::do_off + kk * 2048, L::kRows128, 1024);
                            const uint64_t Qt = sdesc_sw128(sbase + L::q_off + kk * 2048, L::kRows128, 1024);
                            const uint64_t Ph = sdesc_sw128(sbase + L::p_off + kk * 2048, L::kRows128, 1024);
                            const uint64_t Pl =
                                sdesc_sw128(sbase + L::p_off + L::kRows128 + kk * 2048, L::kRows128, 1024);
                            const uint64_t Sh = sdesc_sw128(sbase + L::ds_off + kk * 2048, L::kRows128, 1024);
                            const uint64_t Sl =
                                sdesc_sw128(sbase + L::ds_off + L::kRows128 + kk * 2048, L::kRows128, 1024);
                            mma_ss(tmem + kColDV, dOt, Ph, id_kv, kk > 0);
                            mma_ss(tmem + kColDV, dOt, Pl, id_kv, true);
                            mma_ss(tmem + kColDK, Qt, Sh, id_kv, kk > 0);
                            mma_ss(tmem + kColDK, Qt, Sl, id_kv, true);
                        }
                    }
                    mma_commit(bar_mm2);
                    mma_commit(bar_empty(s));
                    if (t == m.nt - 1) mma_commit(bar_qfree);          // Q / dO of this item no longer read
                    if (t + 2 < m.nt && !(ok = issue_sdp(gtt + 2))) break;
                }
            }
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            gt += m.nt;
        }
        if (!ok) s_abort = 1;
        if (lane == 0) {
            // Every MMA issued is complete before tensor memory is released.
            mma_commit(bar_final);
            mbar_wait(bar_final, 0, kSiteFinal);
        }
    } else {
        // ------------- P and dS, then the dK / dV atomics and the dQ epilogue
        // Thread (warp w, lane l): query row r = 32*(w%4) + l of the M-tile
        // (its tensor-memory lane) and the 16-key quarter kq = w/4 of each tile.
        const int r = (warp % 4) * 32 + lane, kq = warp / 4;
        const int i = r & 63, hp = r >> 6;
        const uint32_t lane_off = uint32_t((warp % 4) * 32) << 16;
        uint8_t* prow_hi = smem + L::p_off + r * 128;
        uint8_t* prow_lo = prow_hi + L::kRows128;
        uint8_t* srow_hi = smem + L::ds_off + r * 128;
        uint8_t* srow_lo = srow_hi + L::kRows128;
        // dV^T / dK^T of tile te of item m (d = tensor-memory lane r, keys of
        // quarter kq) added to the segment's rows; history keys and padding
        // are skipped.
        auto dkv_epilogue = [&](const Item& m, int te) {
            if (!item_tile_has_segment_keys(m, te, a.T_hist)) return;
            tc_fence_after();
            uint32_t vv[16], kv[16];
            tmem_ld16(tmem + lane_off + kColDV + 16 * kq, vv);
            tmem_ld16(tmem + lane_off + kColDK + 16 * kq, kv);
            tmem_wait_ld();
            const bool own = te == m.n_rt;
            int64_t gbase[2];                               // first token of each group slot
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int gi = te * 8 + 2 * kq + q;
                gbase[q] = own ? m.own_start + 16 * kq + 8 * q : (gi < m.n_g ? (int64_t)__ldg(m.grow + gi) * 8 : -64);
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int64_t key = gbase[j / 8] + j % 8;
                if (key < a.T_hist) continue;               // padding or detached history
                const int64_t o = (m.bg * a.T_seg + (key - a.T_hist)) * D + r;
                atomicAdd(a.dV + o, __uint_as_float(vv[j]));
                atomicAdd(a.dK + o, __uint_as_float(kv[j]) * a.scale);
            }
        };
        // Per-row constants of an item.
        struct RowInfo { int64_t row; bool ok; float lse2, Dr; };
        auto row_info = [&](const Item& m) {
            RowInfo ri;
            const int head = m.head0 + hp;
            ri.ok = head < a.G;
            ri.row = (m.b * a.Hq + m.g * a.G + head) * a.T_seg + m.qb * 64 + i;
            ri.lse2 = ri.ok ? __ldg(a.lse + ri.row) * kLog2e : 0.f;
            ri.Dr = ri.ok ? __ldg(a.Drow + ri.row) : 0.f;
            return ri;
        };
        // dQ staging: the P / dS region (64 KB) is free once an item's last
        // MMAs are done; rows of 512 B, 16-byte chunks XOR-swizzled by row.
        float* stage = reinterpret_cast<float*>(smem + L::p_off);
        uint32_t gt = 0;
        bool ok = true;
        int k = 0;
        int64_t it = blockIdx.x;
        Item m = make_item(a, it < n_items ? it : 0, lane);
        RowInfo ri = row_info(m);
        for (; it < n_items && ok; ++k) {
            const int64_t row = ri.row;
            const bool row_ok = ri.ok;
            const float lse2 = ri.lse2, Dr = ri.Dr;
            for (int t = 0; t < m.nt && ok; ++t) {
                const uint32_t gtt = gt + t;
                const int bb = gtt & 1;
                ok = mbar_wait(bar_sdp(bb), (gtt / 2) & 1, kSiteSdp);
                if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
                tc_fence_after();
                const bool own = t == m.n_rt;
                // P is an MMA operand only for dV, i.e. for tiles holding segment keys.
                const bool seg = item_tile_has_segment_keys(m, t, a.T_hist);
                uint32_t sr[16], pr[16];
                tmem_ld16(tmem + lane_off + kColS + bb * kKeys + 16 * kq, sr);
                tmem_ld16(tmem + lane_off + kColDP + bb * kKeys + 16 * kq, pr);
                tmem_wait_ld();
                uint32_t ph[8], pl[8], dh[8], dl[8];
                // Every key of a full routed tile is valid for every row:
                // no masks there; partial tiles and the own chunk mask keys.
                const bool full = row_ok && !own && t * 8 + 8 <= m.n_g;
                const float2 c2 = make_float2(a.scale_log2, a.scale_log2);
                const float2 l2 = make_float2(-lse2, -lse2), d2 = make_float2(-Dr, -Dr);
#pragma unroll
                for (int j2 = 0; j2 < 8; ++j2) {
                    const int j0 = 16 * kq + 2 * j2;
                    const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[2 * j2]), __uint_as_float(sr[2 * j2 + 1])),
                                                c2, l2);
                    float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                    if (!full) {
                        const bool v0 = row_ok && (own ? (j0 <= i) : (t * 8 + j0 / 8 < m.n_g));
                        const bool v1 = row_ok && (own ? (j0 + 1 <= i) : (t * 8 + (j0 + 1) / 8 < m.n_g));
                        p.x = v0 ? p.x : 0.f;
                        p.y = v1 ? p.y : 0.f;
                    }
                    const float2 ds = __fmul2_rn(
                        p, __fadd2_rn(make_float2(__uint_as_float(pr[2 * j2]), __uint_as_float(pr[2 * j2 + 1])), d2));
                    split_bf16x2(ds.x, ds.y, dh[j2], dl[j2]);
                    if (seg) split_bf16x2(p.x, p.y, ph[j2], pl[j2]);
                }
                // The previous tile's MMAs read P / dS from shared memory.
                if (gtt >= 1) {
                    ok = mbar_wait(bar_mm2, (gtt - 1) & 1, kSiteMm2);
                    if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
                }
                // Row r, 16-byte chunk c lives at chunk c ^ (r % 8) (128-byte swizzle).
#pragma unroll
                for (int c2i = 0; c2i < 2; ++c2i) {
                    const int pc = ((2 * kq + c2i) ^ (r & 7)) * 16;
                    *reinterpret_cast<uint4*>(srow_hi + pc) = make_uint4(dh[4 * c2i], dh[4 * c2i + 1], dh[4 * c2i + 2], dh[4 * c2i + 3]);
                    *reinterpret_cast<uint4*>(srow_lo + pc) = make_uint4(dl[4 * c2i], dl[4 * c2i + 1], dl[4 * c2i + 2], dl[4 * c2i + 3]);
                    if (seg) {
                        *reinterpret_cast<uint4*>(prow_hi + pc) = make_uint4(ph[4 * c2i], ph[4 * c2i + 1], ph[4 * c2i + 2], ph[4 * c2i + 3]);
                        *reinterpret_cast<uint4*>(prow_lo + pc) = make_uint4(pl[4 * c2i], pl[4 * c2i + 1], pl[4 * c2i + 2], pl[4 * c2i + 3]);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(bar_ps);
                // While the MMAs of tile t run: the dK / dV of tile t-1.
                if (t >= 1) {
                    dkv_epilogue(m, t - 1);
                    tc_fence_before();
                    mbar_arrive(bar_drained);
                }
            }
            if (!ok) break;
            // The next item's index row and row constants load meanwhile.
            const int64_t it_next = it + gridDim.x;
            const Item m_next = make_item(a, it_next < n_items ? it_next : it, lane);
            const RowInfo ri_next = row_info(m_next);
            const uint32_t last = gt + m.nt - 1;
            ok = mbar_wait(bar_mm2, last & 1, kSiteMm2);
            if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
            dkv_epilogue(m, m.nt - 1);
            tc_fence_before();
            mbar_arrive(bar_drained);
            tc_fence_after();
            // dQ (times the softmax scale): tensor memory -> swizzled shared rows.
            {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + kColDQ + 32 * kq, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const int ch = (32 * kq + j) / 4;              // 16-byte chunk of the row
                    const int pch = (ch & ~7) | ((ch ^ r) & 7);
                    *reinterpret_cast<float4*>(stage + r * D + 4 * pch) =
                        make_float4(__uint_as_float(v[j]) * a.scale, __uint_as_float(v[j + 1]) * a.scale,
                                    __uint_as_float(v[j + 2]) * a.scale, __uint_as_float(v[j + 3]) * a.scale);
                }
            }
            tc_fence_before();
            mbar_arrive(bar_dqfree);
            // All compute threads have staged their dQ parts (bounded wait).
            mbar_arrive(bar_stage);
            if (!mbar_wait(bar_stage, (2 * k) & 1, kSiteStage)) { ok = false; break; }
            // Coalesced rows: warp w writes rows w, w+16, ...; lane l the l-th 16 bytes.
            for (int rr = warp; rr < 128; rr += kComputeWarps) {
                const int head = m.head0 + (rr >> 6);
                if (head >= a.G) continue;
                const int64_t grow_ = (m.b * a.Hq + m.g * a.G + head) * a.T_seg + m.qb * 64 + (rr & 63);
                const int pch = (lane & ~7) | ((lane ^ rr) & 7);
                *reinterpret_cast<float4*>(a.dQ + grow_ * D + 4 * lane) =
                    *reinterpret_cast<const float4*>(stage + rr * D + 4 * pch);
            }
            // The staging rows are read before P / dS of the next item reuse them.
            mbar_arrive(bar_stage);
            if (!mbar_wait(bar_stage, (2 * k + 1) & 1, kSiteStage)) { ok = false; break; }
            (void)row;
            gt += m.nt;
            it = it_next;
            m = m_next;
            ri = ri_next;
        }
        if (!ok) s_abort = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// D_row = sum_e dO[row][e] * O[row][e]: one warp per row, 16-byte loads of O
// and 8-byte loads of dO.
__global__ void __launch_bounds__(256)
rowdot_kernel(const float* __restrict__ O, const __nv_bfloat16* __restrict__ dO, float* __restrict__ Drow,
              int64_t rows)
{
    const int64_t row = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float4 o = __ldg(reinterpret_cast<const float4*>(O + row * D) + lane);
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(dO + row * D) + lane);
    float acc = o.x * __uint_as_float(w.x << 16) + o.y * __uint_as_float(w.x & 0xFFFF0000u) +
                o.z * __uint_as_float(w.y << 16) + o.w * __uint_as_float(w.y & 0xFFFF0000u);
    acc = warp_sum(acc);
    if (lane == 0) Drow[row] = acc;
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
    const uint64_t q_rows = (uint64_t)s.B * s.Hq * s.T_seg, kv_rows = (uint64_t)s.B * s.Hkv * s.T;
    return s.dtype == HGA_BF16 && s.d == D && q_rows < (1ull << 31) && kv_rows < (1ull << 31) &&
           tensor_maps_available();
}

cudaError_t launch_attn_bwd_tc(const Shape& s, const void* Q, const void* K, const void* V, const float* O,
                               const float* lse, const void* dO, const int32_t* gidx, float* dQ,
                               float* dK_seg, float* dV_seg, float* Drow, cudaStream_t st)
{
    const int64_t rows = (int64_t)s.B * s.Hq * s.T_seg;
    rowdot_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(O, static_cast<const __nv_bfloat16*>(dO), Drow, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t seg_bytes = sizeof(float) * (size_t)s.B * s.Hkv * s.T_seg * D;
    if ((e = cudaMemsetAsync(dK_seg, 0, seg_bytes, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dV_seg, 0, seg_bytes, st)) != cudaSuccess) return e;
    CUtensorMap tq, tdo, tk8, tv8, tk64, tv64;
    const uint64_t q_rows = (uint64_t)rows, kv_rows = (uint64_t)s.B * s.Hkv * s.T;
    if (!make_bf16_map(&tq, Q, q_rows, D, 64) || !make_bf16_map(&tdo, dO, q_rows, D, 64) ||
        !make_bf16_map(&tk8, K, kv_rows, D, 8) || !make_bf16_map(&tv8, V, kv_rows, D, 8) ||
        !make_bf16_map(&tk64, K, kv_rows, D, 64) || !make_bf16_map(&tv64, V, kv_rows, D, 64))
        return cudaErrorInvalidValue;
    BwdArgs a;
    a.gidx = gidx;
    a.lse = lse;
    a.Drow = Drow;
    a.dQ = dQ;
    a.dK = dK_seg;
    a.dV = dV_seg;
    a.Hq = s.Hq;
    a.Hkv = s.Hkv;
    a.G = s.G;
    a.wg = s.wg;
    a.T_hist = s.T_hist;
    a.T_seg = s.T_seg;
    a.nQB = s.nQB;
    a.q_rows = (int)q_rows;
    a.scale = s.scale;
    a.scale_log2 = s.scale * kLog2e;
    const int smem = BwdSmem::alloc;
    if ((e = cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
        return e;
    a.n_items = (int64_t)s.B * s.Hkv * s.nQB * ((s.G + 1) / 2);
    const int64_t grid = std::min<int64_t>(a.n_items, sm_count());
    attn_bwd_tc_kernel<<<(unsigned)grid, kThreads, smem, st>>>(tq, tdo, tk8, tv8, tk64, tv64, a);
    return cudaGetLastError();
}

}  // namespace hga
