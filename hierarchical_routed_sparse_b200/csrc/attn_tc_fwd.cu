// attn_tc_fwd.cu -- a5 routed attention forward on the tcgen05 tensor cores
// (bf16 inputs, float32 accumulation and softmax).
//
// Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com),
// section "What HGA does differently": after routing, only the exact token
// K/V of the selected groups is loaded for the attention; summaries are never
// attended.  Query i of a block also attends its own chunk up to itself.
//
// One CTA owns one (batch, kv-head, query block) and up to four q-heads of
// that kv-head: their 64-query blocks stacked into M-tiles of 128 rows (two
// heads per tile), which share every key tile.  Key tiles are 64 tokens: 8
// routed groups (8 rows each, one TMA box per group and 64-column half of d)
// or the own chunk (one box).  Per key tile and M-tile:
//     S  = Q K^T            tcgen05.mma  A = Q (smem), B = K (smem) -> TMEM
//     P  = exp2(S*c - m)    softmax warpgroup, row per thread, P -> TMEM as
//                           two bf16 parts hi + lo (P to ~14 bits)
//     O += P V              tcgen05.mma  A = P hi, P lo (TMEM), B = V (smem)
// The running maximum is only moved when a row's maximum grows by more than
// 2^8 (then O is rescaled in TMEM); any fixed reference point gives the same
// O / l, and it spares most rescales.
//
// Warp roles (320 threads): warps 0-3 softmax of M-tile 0, warps 4-7 of
// M-tile 1, warp 8 TMA producer, warp 9 tensor-memory owner and MMA issuer.
// Tensor memory (512 columns): O of each M-tile (D columns), and two S/P
// buffers of 64 columns per M-tile so that S of the next key tile is computed
// while the softmax works on the current one.
#include "hga_internal.cuh"
#include "sm100.cuh"

namespace hga {

namespace {

using namespace sm100;

constexpr int kStages = 3;          // K/V tiles in flight
constexpr int kKeys = 64;           // keys per tile
constexpr int kThreads = 320;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;

// Status codes of the bounded waits (site of the wait that ran out).
enum : int {
    kSiteQ = 101, kSiteFull, kSiteEmpty, kSiteS, kSiteP, kSiteO, kSiteFinal, kSiteDrain, kSiteStage
};

template <int D>
struct FwdSmem {
    static constexpr int H = D / 64;                  // 64-column halves of d
    static constexpr int kQTile = 128 * 128;          // one M-tile half: 128 rows x 128 B
    static constexpr int kKVHalf = kKeys * 128;       // 64 keys x 128 B
    static constexpr int q_off = 0;
    static constexpr int k_off = q_off + 2 * H * kQTile;
    static constexpr int v_off = k_off + kStages * H * kKVHalf;
    static constexpr int bar_off = v_off + kStages * H * kKVHalf;
    // barriers: q, full[S], empty[S], s[2][2], p[2][2], o[2][2], final, stage
    static constexpr int n_bars = 1 + 2 * kStages + 4 + 4 + 4 + 2;
    static constexpr int tmem_slot_off = bar_off + 8 * n_bars;
    static constexpr int bytes = tmem_slot_off + 16;
    static constexpr int alloc = bytes + 1024;        // room to align the base to 1 KB
};

struct FwdArgs {
    const int32_t* gidx;
    float* O;
    float* lse;
    int Hq, Hkv, G, wg;
    int64_t T_hist, T_seg, nQB;
    int q_rows;          // B*Hq*T_seg (rows of the Q map)
    int kv_rows;         // B*Hkv*T
    float scale_log2;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k8,
                   const __grid_constant__ CUtensorMap tm_v8, const __grid_constant__ CUtensorMap tm_k64,
                   const __grid_constant__ CUtensorMap tm_v64, const FwdArgs a)
{
    using L = FwdSmem<D>;
    constexpr int H = L::H;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::bar_off;
    const uint32_t bar_q = bar0;
    auto bar_full = [&](int s) { return bar0 + 8 * (1 + s); };
    auto bar_empty = [&](int s) { return bar0 + 8 * (1 + kStages + s); };
    auto bar_s = [&](int m, int b) { return bar0 + 8 * (1 + 2 * kStages + 2 * m + b); };
    auto bar_p = [&](int m, int b) { return bar0 + 8 * (5 + 2 * kStages + 2 * m + b); };
    auto bar_o = [&](int m, int b) { return bar0 + 8 * (9 + 2 * kStages + 2 * m + b); };
    const uint32_t bar_final = bar0 + 8 * (13 + 2 * kStages);
    const uint32_t bar_stage = bar0 + 8 * (14 + 2 * kStages);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::tmem_slot_off);
    __shared__ int s_abort;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t u = blockIdx.x;                           // ((b*Hkv)+g)*nQB + qb
    const int64_t qb = u % a.nQB, bg = u / a.nQB;
    const int64_t b = bg / a.Hkv, g = bg % a.Hkv;
    const int head0 = 4 * blockIdx.y;                       // first q-head (within kv-head) of this CTA
    const int n_heads = min(4, a.G - head0);
    const int n_mt = (n_heads + 1) / 2;

    const int32_t* grow = a.gidx + u * a.wg;
    __shared__ int s_ng;
    if (threadIdx.x == 0) s_ng = 0;
    __syncthreads();
    // Routed groups form a prefix of the row: count them with one parallel pass.
    {
        int c = 0;
        for (int i = threadIdx.x; i < a.wg; i += kThreads) c += grow[i] >= 0;
        c = __reduce_add_sync(0xFFFFFFFFu, c);
        if (lane == 0 && c) atomicAdd(&s_ng, c);
    }

    if (threadIdx.x == 0) {
        s_abort = 0;
        mbar_init(bar_q, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        for (int m = 0; m < 2; ++m)
            for (int bb = 0; bb < 2; ++bb) {
                mbar_init(bar_s(m, bb), 1);
                mbar_init(bar_p(m, bb), 128);
                mbar_init(bar_o(m, bb), 1);
            }
        mbar_init(bar_final, 1);
        mbar_init(bar_stage, 128 * n_mt);
        fence_mbar_init();
    }
    if (warp == 9) tmem_alloc(smem_u32(tmem_slot), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_g = s_ng;
    const int n_rt = (n_g + 7) / 8;
    const int nt = n_rt + 1;                                // + own chunk tile
    // Column map: O[m] at m*D, S/P[m][b] at 2*D + (2*m + b)*64.
    auto col_o = [&](int m) { return uint32_t(m * D); };
    auto col_s = [&](int m, int bb) { return uint32_t(2 * D + (2 * m + bb) * kKeys); };

    const int64_t kv_base = bg * (a.T_hist + a.T_seg);      // first K/V row of (b, g)

    if (warp == 8) {
        // ------------------------------------------------------------ producer
        // Lane 0 issues the Q boxes and arms the barriers; for a routed tile,
        // lane j < 8 fetches group j's index and issues that group's boxes,
        // so the eight index loads overlap.
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k8);
            prefetch_tmap(&tm_v8);
            prefetch_tmap(&tm_k64);
            prefetch_tmap(&tm_v64);
            mbar_expect_tx(bar_q, n_mt * 2 * H * 64 * 128);
            for (int hh = 0; hh < 2 * n_mt; ++hh) {
                const int head = head0 + hh;
                // A missing head (odd count) is read past the end: zeros.
                const int y = head < a.G ? int((b * a.Hq + g * a.G + head) * a.T_seg + qb * 64) : a.q_rows;
                for (int c = 0; c < H; ++c)
                    tma_load_2d(sbase + L::q_off + ((hh / 2) * H + c) * L::kQTile + (hh % 2) * 64 * 128,
                                &tm_q, 64 * c, y, bar_q);
            }
        }
        for (int t = 0; t < nt; ++t) {
            const int s = t % kStages, r = t / kStages;
            bool ok = true;
            if (lane == 0) {
                ok = t < kStages || mbar_wait(bar_empty(s), (r - 1) & 1, kSiteEmpty);
                if (ok) mbar_expect_tx(bar_full(s), 2 * H * kKeys * 128);
            }
            if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
                s_abort = 1;
                break;
            }
            const uint32_t kdst = sbase + L::k_off + s * H * L::kKVHalf;
            const uint32_t vdst = sbase + L::v_off + s * H * L::kKVHalf;
            if (t < n_rt) {
                if (lane < 8) {
                    const int gi = t * 8 + lane;
                    // Slots past the last routed group repeat group 0: finite
                    // data whose scores the softmax masks out.
                    const int grp = __ldg(grow + (gi < n_g ? gi : 0));
                    const int y = int(kv_base + (int64_t)grp * 8);
                    for (int c = 0; c < H; ++c) {
                        tma_load_2d(kdst + c * L::kKVHalf + lane * 1024, &tm_k8, 64 * c, y, bar_full(s));
                        tma_load_2d(vdst + c * L::kKVHalf + lane * 1024, &tm_v8, 64 * c, y, bar_full(s));
                    }
                }
            } else if (lane == 0) {
                const int y = int(kv_base + a.T_hist + qb * 64);
                for (int c = 0; c < H; ++c) {
                    tma_load_2d(kdst + c * L::kKVHalf, &tm_k64, 64 * c, y, bar_full(s));
                    tma_load_2d(vdst + c * L::kKVHalf, &tm_v64, 64 * c, y, bar_full(s));
                }
            }
            __syncwarp();
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(128, kKeys, 0, 0);
            constexpr uint32_t id_o = idesc_bf16(128, D, 0, 1);
            bool ok = mbar_wait(bar_q, 0, kSiteQ);
            auto issue_s = [&](int t) -> bool {
                const int s = t % kStages;
                if (!mbar_wait(bar_full(s), (t / kStages) & 1, kSiteFull)) return false;
                tc_fence_after();
                for (int m = 0; m < n_mt; ++m) {
                    const int bb = t & 1;
                    // The buffer held P(t-2), read by PV(t-2).
                    if (t >= 2 && !mbar_wait(bar_o(m, bb), ((t - 2) / 2) & 1, kSiteO)) return false;
                    tc_fence_after();
                    // Descriptors of the operand bases, stepped by constants.
                    const uint64_t dq = sdesc_sw128(sbase + L::q_off + m * H * L::kQTile, 16, 1024);
                    const uint64_t dk = sdesc_sw128(sbase + L::k_off + s * H * L::kKVHalf, 16, 1024);
                    const uint32_t ts = tmem + col_s(m, bb);
#pragma unroll
                    for (int kk = 0; kk < 4 * H; ++kk)
                        mma_ss(ts, dq + (((kk / 4) * L::kQTile + (kk % 4) * 32) >> 4),
                               dk + (((kk / 4) * L::kKVHalf + (kk % 4) * 32) >> 4), id_s, kk > 0);
                    mma_commit(bar_s(m, bb));
                }
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int t = 0; ok && t < nt; ++t) {
                if (t + 1 < nt && !(ok = issue_s(t + 1))) break;
                const int s = t % kStages, bb = t & 1;
                for (int m = 0; m < n_mt; ++m) {
                    if (!(ok = mbar_wait(bar_p(m, bb), (t / 2) & 1, kSiteP))) break;
                    tc_fence_after();
                    const uint64_t vd = sdesc_sw128(sbase + L::v_off + s * H * L::kKVHalf, L::kKVHalf, 1024);
                    const uint32_t to = tmem + col_o(m), tp = tmem + col_s(m, bb);
                    const bool acc = t > 0;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        mma_ts(to, tp + kk * 8, vd + (kk * 16 * 128 >> 4), id_o, acc || kk > 0);
                        mma_ts(to, tp + 32 + kk * 8, vd + (kk * 16 * 128 >> 4), id_o, true);
                    }
                    mma_commit(bar_o(m, bb));
                }
                if (!ok) break;
                mma_commit(bar_empty(s));
            }
            if (!ok) s_abort = 1;
            // Every MMA issued is complete before tensor memory is released.
            mma_commit(bar_final);
            mbar_wait(bar_final, 0, kSiteFinal);
        }
    } else if (warp / 4 < n_mt) {
        // ------------------------------------------------ softmax + epilogue
        const int m = warp / 4, r = threadIdx.x % 128;     // row of the M-tile
        const int i = r & 63, hp = r >> 6;                 // query in block, head in pair
        const int head = head0 + 2 * m + hp;
        const uint32_t lane_off = uint32_t((warp % 4) * 32) << 16;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int t = 0; t < nt && ok; ++t) {
            const int bb = t & 1;
            ok = mbar_wait(bar_s(m, bb), (t / 2) & 1, kSiteS);
            if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
            tc_fence_after();
            uint32_t raw[2][32];
            tmem_ld32(tmem + lane_off + col_s(m, bb), raw[0]);
            tmem_ld32(tmem + lane_off + col_s(m, bb) + 32, raw[1]);
            tmem_wait_ld();
            float sv[64];
            float mx = -INFINITY;
            const bool own = t == n_rt;
            // Full routed tiles need no masks; the scale is applied after the
            // maximum (it is positive) and folded into the exponent's FMA.
            const bool full = !own && t * 8 + 8 <= n_g;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                sv[j] = __uint_as_float(raw[j / 32][j % 32]);
                if (!full && !(own ? (j <= i) : (t * 8 + j / 8 < n_g))) sv[j] = -INFINITY;
                mx = fmaxf(mx, sv[j]);
            }
            mx *= a.scale_log2;
            const bool need = mx > m_run + kRescaleLog2;
            if (__any_sync(0xFFFFFFFFu, need)) {
                const float m_new = need ? mx : m_run;
                const float alpha = fast_exp2(m_run - m_new);  // 0 when m_run = -inf
                if (t > 0) {
                    ok = mbar_wait(bar_o(m, (t - 1) & 1), ((t - 1) / 2) & 1, kSiteO);
                    if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t ov[32];
                        tmem_ld32(tmem + lane_off + col_o(m) + 32 * c, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
                        tmem_st32(tmem + lane_off + col_o(m) + 32 * c, ov);
                    }
                    tmem_wait_st();
                }
                l_run *= alpha;
                m_run = m_new;
            }
            // P = hi + lo, both bf16: the two MMAs carry P to ~14 bits, where
            // one bf16 operand alone (8 bits) misses the 2e-3 output bound.
            uint32_t pk_hi[32], pk_lo[32];
            float2 rs = make_float2(0.f, 0.f);
            const float2 c2 = make_float2(a.scale_log2, a.scale_log2), nm = make_float2(-m_run, -m_run);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float2 x = __ffma2_rn(make_float2(sv[2 * j], sv[2 * j + 1]), c2, nm);
                const float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                rs = __fadd2_rn(rs, p);
                split_bf16x2(p.x, p.y, pk_hi[j], pk_lo[j]);
            }
            l_run += rs.x + rs.y;
            tmem_st32(tmem + lane_off + col_s(m, bb), pk_hi);
            tmem_st32(tmem + lane_off + col_s(m, bb) + 32, pk_lo);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p(m, bb));
        }
        if (ok) {
            ok = mbar_wait(bar_o(m, (nt - 1) & 1), ((nt - 1) / 2) & 1, kSiteO);
            if (__any_sync(0xFFFFFFFFu, !ok)) ok = false;
        }
        if (ok) {
            // O = acc / l through a swizzled shared-memory stage (the Q and
            // K/V buffers are free once the last PV is done), then coalesced
            // row stores.  Row rr of the stage is M-tile rr/128, row rr%128.
            tc_fence_after();
            float* stage = reinterpret_cast<float*>(smem + L::q_off);
            const int sr_ = m * 128 + r;
            const float inv = 1.f / l_run;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t ov[32];
                tmem_ld32(tmem + lane_off + col_o(m) + 32 * c, ov);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const int ch = (32 * c + j) / 4;
                    const int pch = (ch & ~7) | ((ch ^ sr_) & 7);
                    *reinterpret_cast<float4*>(stage + sr_ * D + 4 * pch) =
                        make_float4(__uint_as_float(ov[j]) * inv, __uint_as_float(ov[j + 1]) * inv,
                                    __uint_as_float(ov[j + 2]) * inv, __uint_as_float(ov[j + 3]) * inv);
                }
            }
            if (head < a.G) {
                const int64_t row = ((b * a.Hq + g * a.G + head) * a.T_seg + qb * 64 + i);
                a.lse[row] = (m_run + log2f(l_run)) * kLn2;
            }
            // All softmax threads have staged their rows (bounded wait).
            mbar_arrive(bar_stage);
            if (!mbar_wait(bar_stage, 0, kSiteStage)) s_abort = 1;
            constexpr int C4 = D / 4;                      // 16-byte chunks per row
            for (int rr = warp; rr < 128 * n_mt; rr += 4 * n_mt) {
                const int hh = rr / 64;                    // head within the CTA
                const int head_r = head0 + hh;
                if (head_r >= a.G) continue;
                const int64_t grow_ = (b * a.Hq + g * a.G + head_r) * a.T_seg + qb * 64 + (rr & 63);
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
    if (s_abort && warp == 8 && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            // Loads issued for stage s: tiles s, s+S, ... < nt; wait for the last.
            int last = -1;
            for (int t = s; t < nt; t += kStages) last = t;
            if (last >= 0) mbar_wait(bar_full(s), (last / kStages) & 1, kSiteDrain);
        }
        mbar_wait(bar_q, 0, kSiteDrain);
    }
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---- host side -------------------------------------------------------------------------------------
template <int D>
cudaError_t launch(const Shape& s, const void* Q, const void* K, const void* V, const int32_t* gidx,
                   float* O, float* lse, cudaStream_t st)
{
    CUtensorMap tq, tk8, tv8, tk64, tv64;
    const uint64_t q_rows = (uint64_t)s.B * s.Hq * s.T_seg, kv_rows = (uint64_t)s.B * s.Hkv * s.T;
    if (!make_bf16_map(&tq, Q, q_rows, D, 64) || !make_bf16_map(&tk8, K, kv_rows, D, 8) ||
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
    a.scale_log2 = s.scale * kLog2e;
    auto k = attn_fwd_tc_kernel<D>;
    const int smem = FwdSmem<D>::alloc;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(s.B * s.Hkv * s.nQB), (unsigned)((s.G + 3) / 4));
    k<<<grid, kThreads, smem, st>>>(tq, tk8, tv8, tk64, tv64, a);
    return cudaGetLastError();
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
    const uint64_t q_rows = (uint64_t)s.B * s.Hq * s.T_seg, kv_rows = (uint64_t)s.B * s.Hkv * s.T;
    return s.dtype == HGA_BF16 && (s.d == 128 || s.d == 64) && q_rows < (1ull << 31) &&
           kv_rows < (1ull << 31) && tensor_maps_available();
}

cudaError_t launch_attn_fwd_tc(const Shape& s, const void* Q, const void* K, const void* V,
                               const int32_t* gidx, float* O, float* lse, cudaStream_t st)
{
    return s.d == 128 ? launch<128>(s, Q, K, V, gidx, O, lse, st) : launch<64>(s, Q, K, V, gidx, O, lse, st);
}

}  // namespace hga
