// causal.cu -- the strictly causal variant: routing per query position.
//
// Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com),
// section "The one real caveat: causal leakage": with block routing the
// routing of a block depends on the scores of several query positions, so an
// earlier token sees later tokens through it; the authors mention a strictly
// causal variant in the works.  This variant routes every query position on
// its own query -- a query block of one, as the decode step does: the mean of
// its G q-heads' queries scores the chunks before its own chunk (top k_c),
// then the groups of those chunks (top k_g); each q-head attends the routed
// groups' exact tokens and its own chunk up to itself.  The output at a
// position then depends on earlier positions only.
//
// Every row has its own key set, so there is no key tile shared by the rows
// of a block: the kernels work per (row, kv-head) on the FMA pipes.
//   causal_route_win_kernel  one CTA per window of 32 neighbouring positions
//                        of a (batch, kv-head), which share their own chunk
//                        and so their chunk candidates: the chunk scores of
//                        the 32 rows as a register-tiled float32 product
//                        with the chunk summaries staged once in shared
//                        memory, a warp top-k per row, then the group
//                        summaries of the union of the rows' chosen chunks
//                        read once (a chunk per warp, in registers) and
//                        scored against every row that chose the chunk,
//                        warp rank selection;
//   causal_route_kernel  (shapes the window kernel does not take) one warp
//                        per row: block query of one, chunk scores (the 8
//                        rows of a CTA share the summaries through L1), warp
//                        top-k, group scores, warp rank selection;
//   causal_fwd_kernel    one warp per (row, kv-head), the G heads together,
//                        keys in batches of 32: scores with one key per lane
//                        (the lane reads the key's whole K row and dots it
//                        with the G queries held in shared memory), a
//                        running softmax per head, then P V with lanes over
//                        the head dims (V rows in flight, each key's weight
//                        broadcast from its lane); O and lse;
//   causal_bwd_kernel    one warp per (row, kv-head), the same two layouts:
//                        per key P from lse, dP, dS by lanes over keys; dQ
//                        in registers and the key's dK / dV over head dims,
//                        added to the segment's rows with vector float
//                        atomics.
// Float32 arithmetic (packed fp32x2 FMAs); bf16 or float32 inputs.
#include "check.cuh"
#include "hga_internal.cuh"
#include "router_core.cuh"
#include "sm100.cuh"
#include "window_union.cuh"

namespace hga {
namespace {

using namespace rt;
using namespace sm100;

constexpr int kWarps = 8;                   // rows (warps) per CTA
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxG = 8;                    // q-heads per kv-head

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~size_t(15); }

// Per-warp shared memory of the routing kernel.
struct RouteWarpLayout {
    size_t keys, ids, flags, crow, qs, total;
};
__host__ __device__ inline RouteWarpLayout route_warp_layout(int64_t nC, int wc, int D)
{
    RouteWarpLayout L;
    const size_t nk = (size_t)(nC > 8 * (int64_t)wc ? nC : 8 * (int64_t)wc);
    L.keys = 0;
    L.ids = al16(L.keys + 8 * nk);
    L.flags = al16(L.ids + 4 * 8 * (size_t)wc);
    L.crow = al16(L.flags + 8 * (size_t)wc);
    L.qs = al16(L.crow + 4 * (size_t)wc);
    L.total = al16(L.qs + 4 * (size_t)D);
    return L;
}

// P consecutive elements widened to float32 (4- to 16-byte loads).
template <typename TIn, int P> struct Row;
template <> struct Row<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* o) {
        const uint2 r = __ldg(reinterpret_cast<const uint2*>(p));
        o[0] = __uint_as_float(r.x << 16); o[1] = __uint_as_float(r.x & 0xFFFF0000u);
        o[2] = __uint_as_float(r.y << 16); o[3] = __uint_as_float(r.y & 0xFFFF0000u);
    }
};
template <> struct Row<__nv_bfloat16, 2> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* o) {
        const uint32_t r = __ldg(reinterpret_cast<const unsigned int*>(p));
        o[0] = __uint_as_float(r << 16); o[1] = __uint_as_float(r & 0xFFFF0000u);
    }
};
template <> struct Row<float, 4> {
    static __device__ __forceinline__ void load(const float* p, float* o) {
        const float4 r = __ldg(reinterpret_cast<const float4*>(p));
        o[0] = r.x; o[1] = r.y; o[2] = r.z; o[3] = r.w;
    }
};
template <> struct Row<float, 2> {
    static __device__ __forceinline__ void load(const float* p, float* o) {
        const float2 r = __ldg(reinterpret_cast<const float2*>(p));
        o[0] = r.x; o[1] = r.y;
    }
};

// a4 selection inside one warp: of the n scored candidates (keys, ids) keep
// those beaten by fewer than k_g others; kept ids in candidate order to out.
__device__ __forceinline__ void warp_select_groups(unsigned long long* keys, const int32_t* ids, int n, int k_g,
                                                   uint8_t* flags, int32_t* out, int wg, int lane)
{
    for (int i = lane; i < n; i += 32) {
        const unsigned long long ki = keys[i];
        int rank = 0;
        for (int j = 0; j < n; ++j) rank += keys[j] > ki;
        flags[i] = rank < k_g;
    }
    __syncwarp();
    for (int i = lane; i < n; i += 32)
        if (flags[i]) keys[i] = 0ull;
    __syncwarp();
    compact_selected(keys, ids, n, out, wg, lane);
}

// Routing of every query position: warp w of CTA x routes row
// 8 x + w of the (batch, kv-head, row) grid.  cidx [B][Hkv][T_seg][wc],
// gidx [B][Hkv][T_seg][wg].
template <typename TIn, int D>
__global__ void __launch_bounds__(kThreads)
causal_route_kernel(const TIn* __restrict__ Q, const float* __restrict__ csum, const float* __restrict__ gsum,
                    int32_t* __restrict__ cidx, int32_t* __restrict__ gidx, int Hq, int Hkv, int G,
                    int64_t T_hist, int64_t T_seg, int64_t cap, int k_c, int wc, int k_g, int wg)
{
    pdl_wait();
    pdl_trigger();
    constexpr int P = D / 32;
    extern __shared__ __align__(16) uint8_t sm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t T = T_hist + T_seg, nC = T / kChunk, nCs = cap / kChunk, nGs = cap / kGroup;
    const RouteWarpLayout L = route_warp_layout(nC, wc, D);
    uint8_t* ws = sm + (size_t)warp * L.total;
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(ws + L.keys);
    int32_t* ids = reinterpret_cast<int32_t*>(ws + L.ids);
    uint8_t* flags = ws + L.flags;
    int32_t* crow = reinterpret_cast<int32_t*>(ws + L.crow);
    float* qs = reinterpret_cast<float*>(ws + L.qs);
    const int64_t row = (int64_t)blockIdx.x * kWarps + warp;      // (b, g, i) flattened
    const int64_t bg = row / T_seg, i = row % T_seg;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    // Block query of one: the mean of the row's G q-heads' queries.
    float a[P];
#pragma unroll
    for (int e = 0; e < P; ++e) a[e] = 0.f;
    for (int h = 0; h < G; ++h) {
        float x[P];
        Row<TIn, P>::load(Q + ((b * Hq + g * G + h) * T_seg + i) * D + lane * P, x);
#pragma unroll
        for (int e = 0; e < P; ++e) a[e] += x[e];
    }
#pragma unroll
    for (int e = 0; e < P; ++e) qs[lane * P + e] = a[e] / (float)G;
    __syncwarp();
    // a3: chunks before the row's own chunk.
    const int c0 = int((T_hist + i) / kChunk);
    int32_t* crow_out = cidx + row * wc;
    if (k_c <= 0 || k_c >= c0) {
        for (int j = lane; j < wc; j += 32) {
            const int32_t v = j < c0 ? j : -1;
            crow[j] = v;
            crow_out[j] = v;
        }
    } else {
        const float* cs = csum + bg * nCs * D;
        score_candidates<D, 1>(qs, c0, [&](int c, const float*& r) { r = cs + (int64_t)c * D; return c; }, keys, 0,
                               lane);
        __syncwarp();
        select_chunks(keys, c0, k_c, wc, crow, crow_out, 0, lane);
    }
    __syncwarp();
    // a4: the groups of the chosen chunks.
    const int n = prefix_count(crow, wc, lane) * kGroupsPerChunk;
    for (int j = lane; j < n; j += 32) ids[j] = crow[j / kGroupsPerChunk] * kGroupsPerChunk + j % kGroupsPerChunk;
    __syncwarp();
    int32_t* grow_out = gidx + row * wg;
    if (k_g <= 0 || k_g >= n) {
        for (int j = lane; j < wg; j += 32) grow_out[j] = j < n ? ids[j] : -1;
    } else {
        const float* gs = gsum + bg * nGs * D;
        score_candidates<D, 1>(qs, n, [&](int c, const float*& r) { r = gs + (int64_t)ids[c] * D; return ids[c]; },
                               keys, 0, lane);
        __syncwarp();
        warp_select_groups(keys, ids, n, k_g, flags, grow_out, wg, lane);
    }
}

// ---- windowed routing ------------------------------------------------------------------------
// The 32 positions of a window lie in one chunk, so all have the same chunk
// candidates (c < own chunk): their chunk scores are a [32 x c0] product of
// the rows' block queries with the chunk summaries, computed in tiles of 256
// chunks, whose summaries stream through shared memory in slices of 16 dims
// (asynchronous copies, two buffers: slice s + 1 lands while slice s is
// used).  Warp w covers rows 16 (w & 1) .. + 15 and chunks 64 (w >> 1) ..
// + 63 of a tile; lane (tr, tc) = (lane >> 3, lane & 7) rows 16 (w & 1) +
// tr + 4 i (i < 4) and chunks 64 (w >> 1) + tc + 8 j (j < 8).  Each score is one float32 chain
// over the head dims in order.  Then the group summaries of the union of
// the rows' chosen chunks are read once per window, a chunk per warp held in
// registers, and scored against every row that chose the chunk.
namespace rwin {
constexpr int kW = 32;              // positions of a window
constexpr int kWinThreads = 256;
constexpr int kCT = 256;            // chunks of a score tile
constexpr int kDS = 16;             // head dims of a staged summary slice
constexpr int kRowsPerWarp = kW / (kWinThreads / 32);
}  // namespace rwin

struct WinLayout {
    size_t q, c, s, crow, uni, total;
    int sstride, gkeys, gids, gflags;   // offsets inside the S region (group stage)
    int nwords;                         // bitmap words over the context's chunks
};
__host__ __device__ inline WinLayout win_layout(int64_t nC, int wc, int D)
{
    using namespace rwin;
    WinLayout L;
    const size_t qs = (size_t)D + 4;
    L.q = 0;                                                       // block queries [kW][D + 4]
    L.c = al16(L.q + 4 * kW * qs);                                 // two summary slices
    const size_t cbytes = 2 * 4 * (size_t)kCT * (kDS + 4);
    L.sstride = int((nC + 3) & ~int64_t(3));                       // chunk scores [kW][sstride]
    const size_t ng = 8 * (size_t)wc;
    // Group stage, in the same region: scores [kW][8 wc], then per warp the
    // keys (8 B), ids (4 B) and flags (1 B) of 8 wc candidates.
    constexpr int nwarps = kWinThreads / 32;
    L.gkeys = int(al16(4 * kW * ng));
    L.gids = int(L.gkeys + nwarps * 8 * ng);
    L.gflags = int(L.gids + nwarps * 4 * ng);
    const size_t sb = 4 * (size_t)kW * L.sstride, gsz = L.gflags + nwarps * al16(ng);
    const size_t sreg = sb > gsz ? sb : gsz;
    if (nC - 1 <= kCT) {
        // One score tile (c0 <= 256): the scores are written after its last
        // slice is consumed, so they (and the group stage) reuse the slices.
        L.s = L.c;
        L.crow = al16(L.c + (cbytes > sreg ? cbytes : sreg));
    } else {
        L.s = al16(L.c + cbytes);
        L.crow = al16(L.s + sreg);
    }
    L.uni = al16(L.crow + 4 * (size_t)kW * wc);                    // chosen chunks [kW][wc]
    L.nwords = int((nC + 31) / 32);                                // union: bitmap, prefix, list, masks, count
    L.total = al16(L.uni + 8 * (size_t)L.nwords + 8 * (size_t)kW * wc + 16 + (size_t)kW * kW * wc);
    return L;
}

// Top-k of the float scores s[0..n) (n <= 2048), "higher score, then lower
// index", written ascending to out0 and out1, -1 up to `width`.  Lane l
// owns candidates l + 32 m and marks its selected ones in a 64-bit mask.
__device__ __forceinline__ void topk_scores_rounds(const float* s, int n, int k, int32_t* out0, int32_t* out1,
                                                   int width, int lane)
{
    uint64_t sel = 0;
    auto best_of = [&]() {
        unsigned long long b = 0ull;
        for (int m = 0, c = lane; c < n; ++m, c += 32)
            if (!((sel >> m) & 1ull)) {
                const unsigned long long kc = pack_key(s[c], c);
                b = kc > b ? kc : b;
            }
        return b;
    };
    unsigned long long best = best_of();
    for (int round = 0; round < k; ++round) {
        const uint32_t hi = uint32_t(best >> 32), lo = uint32_t(best);
        const uint32_t mhi = __reduce_max_sync(0xFFFFFFFFu, hi);
        const uint32_t mlo = __reduce_max_sync(0xFFFFFFFFu, hi == mhi ? lo : 0u);
        if (best != 0ull && hi == mhi && lo == mlo) {   // keys are distinct: one lane wins
            sel |= 1ull << (key_index(best) >> 5);
            best = best_of();
        }
    }
    const unsigned below = (1u << lane) - 1u;
    int pos = 0;
    for (int m = 0; 32 * m < n; ++m) {
        const bool mine = (sel >> m) & 1ull;
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, mine);
        if (mine) {
            const int at = pos + __popc(bal & below);
            out0[at] = lane + 32 * m;
            out1[at] = lane + 32 * m;
        }
        pos += __popc(bal);
    }
    for (int i = pos + lane; i < width; i += 32) {
        out0[i] = -1;
        out1[i] = -1;
    }
}

// Sorted (descending) list of the 8 largest keys seen by a lane.
struct Top8 {
    unsigned long long v[8];
    __device__ __forceinline__ void init()
    {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0ull;
    }
    __device__ __forceinline__ void push(unsigned long long x)
    {
        if (x <= v[7]) return;
        v[7] = x;
#pragma unroll
        for (int i = 7; i > 0; --i)
            if (v[i] > v[i - 1]) {
                const unsigned long long t = v[i];
                v[i] = v[i - 1];
                v[i - 1] = t;
            }
    }
    // Keep the 8 largest of this list and the list of lane ^ o (both
    // sorted): the element-wise maximum against the partner's list reversed
    // is a bitonic sequence holding them, sorted again by a bitonic merge.
    __device__ __forceinline__ void merge_xor(int o)
    {
        unsigned long long p[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) p[i] = __shfl_xor_sync(0xFFFFFFFFu, v[i], o);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = v[i] > p[7 - i] ? v[i] : p[7 - i];
#pragma unroll
        for (int d = 4; d > 0; d >>= 1)
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if ((i & d) == 0 && v[i + d] > v[i]) {
                    const unsigned long long t = v[i];
                    v[i] = v[i + d];
                    v[i + d] = t;
                }
    }
};

// Top-k (k <= 8) of the float scores s[0..n) by key ("higher score, then
// lower index"), for one row per group of 8 lanes (sub = lane & 7): each
// lane keeps the 8 best of candidates sub, sub + 8, ..., the group merges
// them, and lane sub writes slot sub of the row (ascending chunk indices,
// -1 past k) to out0 and out1 (width <= 8).
__device__ __forceinline__ void topk8_lanes(const float* s, int n, int k, int32_t* out0, int32_t* out1, int width,
                                            int sub)
{
    Top8 t;
    t.init();
    for (int c = sub; c < n; c += 8) t.push(pack_key(s[c], c));
    t.merge_xor(1);
    t.merge_xor(2);
    t.merge_xor(4);
    int idx[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) idx[i] = i < k ? key_index(t.v[i]) : INT32_MAX;
#pragma unroll
    for (int a = 0; a < 8; ++a)                       // ascending (a small sort network would do too)
#pragma unroll
        for (int b = 0; b < 7 - a; ++b)
            if (idx[b] > idx[b + 1]) {
                const int x = idx[b];
                idx[b] = idx[b + 1];
                idx[b + 1] = x;
            }
    int mine = -1;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (i == sub) mine = idx[i] == INT32_MAX ? -1 : idx[i];
    if (sub < width) {
        out0[sub] = mine;
        out1[sub] = mine;
    }
}

// Group top-k over n <= 64 candidate keys (keys[0..n), ids; one warp):
// the k-th largest key by a bitonic sort of the 64 (lane holds elements
// lane and lane + 32), then the candidates with a key at least that large
// are written in candidate order, -1 up to `width`.
__device__ __forceinline__ void select_groups64(const unsigned long long* keys, const int32_t* ids, int n, int k,
                                               int32_t* out, int width, int lane)
{
    unsigned long long a = lane < n ? keys[lane] : 0ull, b = lane + 32 < n ? keys[lane + 32] : 0ull;
#pragma unroll
    for (int sz = 2; sz <= 64; sz <<= 1) {
#pragma unroll
        for (int j = sz >> 1; j > 0; j >>= 1) {
            if (j == 32) {                                   // elements lane and lane + 32: descending
                const unsigned long long hi = a > b ? a : b, lo = a > b ? b : a;
                a = hi;
                b = lo;
                continue;
            }
            const bool lower = (lane & j) == 0;
            const bool desc_a = sz == 64 || (lane & sz) == 0;
            const bool desc_b = sz == 64 || ((lane + 32) & sz) == 0;
            const unsigned long long pa = __shfl_xor_sync(0xFFFFFFFFu, a, j);
            const unsigned long long pb = __shfl_xor_sync(0xFFFFFFFFu, b, j);
            a = (lower == desc_a) ? (a > pa ? a : pa) : (a < pa ? a : pa);
            b = (lower == desc_b) ? (b > pb ? b : pb) : (b < pb ? b : pb);
        }
    }
    const int e = k - 1;                                     // descending: position k - 1
    const unsigned long long kth = __shfl_sync(0xFFFFFFFFu, e < 32 ? a : b, e & 31);
    const unsigned below = (1u << lane) - 1u;
    int pos = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int j = lane + 32 * h;
        const bool sel = j < n && keys[j] >= kth;
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) out[pos + __popc(bal & below)] = ids[j];
        pos += __popc(bal);
    }
    for (int i = pos + lane; i < width; i += 32) out[i] = -1;
}

// CTA x routes positions w0 .. w0 + 31 of (batch, kv-head) x / (T_seg / 32).
template <typename TIn, int D>
__global__ void __launch_bounds__(rwin::kWinThreads, 2)
causal_route_win_kernel(const TIn* __restrict__ Q, const float* __restrict__ csum, const float* __restrict__ gsum,
                        int32_t* __restrict__ cidx, int32_t* __restrict__ gidx, int Hq, int Hkv, int G,
                        int64_t T_hist, int64_t T_seg, int64_t cap, int k_c, int wc, int k_g, int wg)
{
    using namespace rwin;
    pdl_wait();
    pdl_trigger();
    constexpr int P = D / 32, QS = D + 4, CS = kDS + 4;
    extern __shared__ __align__(16) uint8_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t T = T_hist + T_seg, nC = T / kChunk, nCs = cap / kChunk, nGs = cap / kGroup;
    const WinLayout L = win_layout(nC, wc, D);
    float* q_s = reinterpret_cast<float*>(sm + L.q);
    float* c_s = reinterpret_cast<float*>(sm + L.c);
    float* S = reinterpret_cast<float*>(sm + L.s);
    int32_t* crow_s = reinterpret_cast<int32_t*>(sm + L.crow);
    const int SS = L.sstride;
    const int64_t nWin = T_seg / kW;
    const int64_t bg = blockIdx.x / nWin, w0 = (blockIdx.x % nWin) * kW;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    const int c0 = int((T_hist + w0) / kChunk);               // own chunk of every row of the window
    // Block queries of one: the mean of each row's G q-heads' queries, a
    // row's loads issued before its sums.
#pragma unroll 1
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int r = warp * kRowsPerWarp + rr;
        float x[kMaxG][P];
#pragma unroll
        for (int h = 0; h < kMaxG; ++h)
            if (h < G) Row<TIn, P>::load(Q + ((b * Hq + g * G + h) * T_seg + w0 + r) * D + lane * P, x[h]);
        float a[P];
#pragma unroll
        for (int e = 0; e < P; ++e) a[e] = 0.f;
#pragma unroll
        for (int h = 0; h < kMaxG; ++h)
            if (h < G)
#pragma unroll
                for (int e = 0; e < P; ++e) a[e] += x[h][e];
#pragma unroll
        for (int e = 0; e < P; ++e) q_s[r * QS + lane * P + e] = a[e] / (float)G;
    }
    __syncthreads();
    // a3: chunk scores of the rows, then a top-k_c per row.
    const bool all_c = k_c <= 0 || k_c >= c0;
    if (!all_c) {
        const float* cs = csum + bg * nCs * D;
        const int rh = warp & 1, cq = warp >> 1, tr = lane >> 3, tc = lane & 7;
        const uint32_t cbase = smem_u32(c_s);
        constexpr int NS = D / kDS;                            // slices of a tile
        constexpr int kCopies = kCT * (kDS / 4) / kWinThreads; // 16-byte copies per thread and slice
        // Slice ds of chunks ct0 .. ct0 + nct into buffer `buf` (zeros past nct).
        auto issue = [&](int ct0, int nct, int ds, int buf) {
#pragma unroll
            for (int k = 0; k < kCopies; ++k) {
                const int idx = tid + k * kWinThreads;
                const int c = idx / (kDS / 4), v = idx % (kDS / 4);
                const bool valid = c < nct;
                cp_async16(cbase + 4u * uint32_t(buf * kCT * CS + c * CS + 4 * v),
                           cs + (int64_t)(valid ? ct0 + c : 0) * D + ds + 4 * v, valid);
            }
            cp_async_commit();
        };
        for (int ct0 = 0; ct0 < c0; ct0 += kCT) {
            const int nct = min(kCT, c0 - ct0);
            float acc[4][8];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
            issue(ct0, nct, 0, 0);
            for (int si = 0; si < NS; ++si) {
                if (si + 1 < NS) {
                    issue(ct0, nct, (si + 1) * kDS, (si + 1) & 1);   // its buffer's last reader synced below
                    cp_async_wait<1>();
                } else {
                    cp_async_wait<0>();
                }
                __syncthreads();                               // slice si has landed for every thread
                const float* cb = c_s + (si & 1) * kCT * CS;
                const int ds = si * kDS;
#pragma unroll
                for (int e4 = 0; e4 < kDS / 4; ++e4) {
                    float4 qv[4], cv[8];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        qv[i] = *reinterpret_cast<const float4*>(q_s + (16 * rh + tr + 4 * i) * QS + ds + 4 * e4);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        cv[j] = *reinterpret_cast<const float4*>(cb + (64 * cq + tc + 8 * j) * CS + 4 * e4);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            float t = fmaf(qv[i].x, cv[j].x, acc[i][j]);
                            t = fmaf(qv[i].y, cv[j].y, t);
                            t = fmaf(qv[i].z, cv[j].z, t);
                            acc[i][j] = fmaf(qv[i].w, cv[j].w, t);
                        }
                }
                __syncthreads();                               // buffer si & 1 free for slice si + 2
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int c = 64 * cq + tc + 8 * j;
                    if (c < nct) S[(16 * rh + tr + 4 * i) * SS + ct0 + c] = acc[i][j];
                }
        }
        __syncthreads();
    }
    if (!all_c && k_c <= 8) {
        // Eight lanes per row: the warp's four rows at once.
        const int r = warp * kRowsPerWarp + (lane >> 3);
        topk8_lanes(S + r * SS, c0, k_c, crow_s + r * wc, cidx + (bg * T_seg + w0 + r) * wc, wc, lane & 7);
    } else
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int r = warp * kRowsPerWarp + rr;
        int32_t* out = cidx + (bg * T_seg + w0 + r) * wc;
        int32_t* crow = crow_s + r * wc;
        if (all_c) {
            for (int j = lane; j < wc; j += 32) {
                const int32_t v = j < c0 ? j : -1;
                crow[j] = v;
                out[j] = v;
            }
        } else if (c0 <= 32 * kRegCand) {
            unsigned long long ck[kRegCand];
#pragma unroll
            for (int m = 0; m < kRegCand; ++m) {
                const int c = lane + 32 * m;
                ck[m] = c < c0 ? pack_key(S[r * SS + c], c) : 0ull;
            }
            warp_topk_regs(ck, k_c, crow, out, wc, lane);
        } else {
            topk_scores_rounds(S + r * SS, c0, k_c, crow, out, wc, lane);
        }
    }
    __syncthreads();
    // a4: the groups of each row's chosen chunks.
    const bool all_g = k_g <= 0 || k_g >= 8 * wc;              // every row keeps all its candidates
    const int ng = 8 * wc;
    float* Sg = S;                                             // [kW][8 wc] group scores (chunk scores done)
    if (!all_g) {
        // The union of the rows' chosen chunks (bitmap, prefix ranks, the
        // ascending list) and per union chunk the mask of the rows that
        // chose it.
        uint32_t* bitmap = reinterpret_cast<uint32_t*>(sm + L.uni);
        uint32_t* prefix = bitmap + L.nwords;
        int32_t* ulist = reinterpret_cast<int32_t*>(prefix + L.nwords);
        uint32_t* umask = reinterpret_cast<uint32_t*>(ulist + kW * wc);
        int* s_u = reinterpret_cast<int*>(umask + kW * wc);
        uint8_t* uslot = reinterpret_cast<uint8_t*>(s_u + 4);   // [union chunk][row]: the chunk's slot in the row
        const int nwc = (c0 + 31) / 32;
        for (int i = tid; i < nwc; i += kWinThreads) bitmap[i] = 0u;
        for (int i = tid; i < kW * wc; i += kWinThreads) umask[i] = 0u;
        __syncthreads();
        for (int e = tid; e < kW * wc; e += kWinThreads) {
            const int c = crow_s[e];
            if (c >= 0) atomicOr(&bitmap[c >> 5], 1u << (c & 31));
        }
        __syncthreads();
        if (warp == 0) {
            int run = 0;
            for (int base = 0; base < nwc; base += 32) {
                const int wd = base + lane;
                const int cnt = wd < nwc ? __popc(bitmap[wd]) : 0;
                int incl = cnt;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (wd < nwc) prefix[wd] = uint32_t(run + incl - cnt);
                run += __shfl_sync(0xFFFFFFFFu, incl, 31);
            }
            if (lane == 0) *s_u = run;
        }
        __syncthreads();
        for (int wd = tid; wd < nwc; wd += kWinThreads) {
            uint32_t word = bitmap[wd];
            int k = int(prefix[wd]);
            while (word) {
                ulist[k++] = wd * 32 + __ffs(word) - 1;
                word &= word - 1;
            }
        }
        for (int e = tid; e < kW * wc; e += kWinThreads) {
            const int c = crow_s[e];
            if (c < 0) continue;
            const int rank = int(prefix[c >> 5]) + __popc(bitmap[c >> 5] & ((1u << (c & 31)) - 1u));
            atomicOr(&umask[rank], 1u << (e / wc));
            uslot[rank * kW + e / wc] = uint8_t(e % wc);
        }
        __syncthreads();
        // Warp w takes union chunks w, w + 8, ...: lane (gl, sq) holds group
        // gl's head dims 4 (sq + 4 j) .. + 3 of the chunk in registers (the
        // next chunk's loads in flight meanwhile), and for every row that
        // chose the chunk dots them with the row's block query; the four
        // quarters are summed across the warp.  Each group summary is read
        // once per window.
        const int U = *s_u;
        const float* gs = gsum + bg * nGs * D;
        const int gl = lane & 7, sq = lane >> 3;
        constexpr int J = D / 16;
        float4 cur[J], nxt[J];
        auto load_chunk = [&](int u, float4 (&v)[J]) {
            const float4* grow =
                reinterpret_cast<const float4*>(gs + ((int64_t)ulist[u] * kGroupsPerChunk + gl) * D);
#pragma unroll
            for (int j = 0; j < J; ++j) v[j] = __ldg(grow + sq + 4 * j);
        };
        if (warp < U) load_chunk(warp, cur);
        for (int u = warp; u < U; u += kWinThreads / 32) {
            if (u + kWinThreads / 32 < U) load_chunk(u + kWinThreads / 32, nxt);
            uint32_t m = umask[u];
            while (m) {                                        // the same for the whole warp
                const int r = __ffs(m) - 1;
                m &= m - 1;
                const int k = uslot[u * kW + r];
                const float* qrow = q_s + r * QS;
                float a = 0.f;
#pragma unroll
                for (int j = 0; j < J; ++j) {
                    const float4 qv = *reinterpret_cast<const float4*>(qrow + 4 * (sq + 4 * j));
                    a = fmaf(qv.x, cur[j].x, a);
                    a = fmaf(qv.y, cur[j].y, a);
                    a = fmaf(qv.z, cur[j].z, a);
                    a = fmaf(qv.w, cur[j].w, a);
                }
                a += __shfl_xor_sync(0xFFFFFFFFu, a, 8);
                a += __shfl_xor_sync(0xFFFFFFFFu, a, 16);
                if (sq == 0) Sg[r * ng + 8 * k + gl] = a;
            }
#pragma unroll
            for (int j = 0; j < J; ++j) cur[j] = nxt[j];
        }
        __syncthreads();                                       // every row's scores are in
    }
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(sm + L.s + L.gkeys) + (size_t)warp * ng;
    int32_t* ids = reinterpret_cast<int32_t*>(sm + L.s + L.gids) + (size_t)warp * ng;
    uint8_t* flags = sm + L.s + L.gflags + (size_t)warp * al16(ng);
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int r = warp * kRowsPerWarp + rr;
        int32_t* gout = gidx + (bg * T_seg + w0 + r) * wg;
        const int n = prefix_count(crow_s + r * wc, wc, lane) * kGroupsPerChunk;
        for (int j = lane; j < n; j += 32) ids[j] = crow_s[r * wc + j / 8] * kGroupsPerChunk + j % 8;
        __syncwarp();
        if (k_g <= 0 || k_g >= n) {
            for (int j = lane; j < wg; j += 32) gout[j] = j < n ? ids[j] : -1;
        } else {
            for (int j = lane; j < n; j += 32) keys[j] = pack_key(Sg[r * ng + j], ids[j]);
            __syncwarp();
            if (n <= 64) select_groups64(keys, ids, n, k_g, gout, wg, lane);
            else warp_select_groups(keys, ids, n, k_g, flags, gout, wg, lane);
        }
        __syncwarp();
    }
}

// Key k of a row: the routed groups' tokens in order, then the own chunk's
// tokens own0 .. pos.
__device__ __forceinline__ int64_t row_token(const int32_t* grow, int n_g, int64_t own0, int k, int site)
{
    return k < kGroup * n_g ? (int64_t)chk::group(__ldg(grow + k / kGroup), own0 / kGroup, site) * kGroup + k % kGroup
                            : own0 + (k - kGroup * n_g);
}

// 16 bytes of a row widened to float32 (8 bf16 or 4 float).
template <typename TIn> struct U4;
template <> struct U4<__nv_bfloat16> {
    static constexpr int E = 8;
    static __device__ __forceinline__ void unpack(const uint4& r, float* x) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <> struct U4<float> {
    static constexpr int E = 4;
    static __device__ __forceinline__ void unpack(const uint4& r, float* x) {
        x[0] = __uint_as_float(r.x); x[1] = __uint_as_float(r.y);
        x[2] = __uint_as_float(r.z); x[3] = __uint_as_float(r.w);
    }
};

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// s2[h] += x . rows[h][e0 .. e0+E) of the G rows held in shared memory
// (floats, row stride D), for 16 bytes of a key row widened to x; packed
// fp32x2 FMAs, the even and odd elements in the two halves of s2[h].
template <typename TIn, int D, int GM>
__device__ __forceinline__ void dot16(const float* rows, int G, int e0, const uint4& raw, float2* s2)
{
    constexpr int E = U4<TIn>::E;
    float x[E];
    U4<TIn>::unpack(raw, x);
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        if (h >= G) break;
#pragma unroll
        for (int v = 0; v < E; v += 4) {
            const float4 q = *reinterpret_cast<const float4*>(rows + h * D + e0 + v);
            s2[h] = __ffma2_rn(make_float2(q.x, q.y), make_float2(x[v], x[v + 1]), s2[h]);
            s2[h] = __ffma2_rn(make_float2(q.z, q.w), make_float2(x[v + 2], x[v + 3]), s2[h]);
        }
    }
}

// s[h] = rows[h] . key row (all D elements), the key row read by this lane
// alone in pieces of MaxInFlight loads of 16 bytes, each piece all in flight.
template <typename TIn, int D, int GM, int MaxInFlight = 16>
__device__ __forceinline__ void row_dots(const float* rows, int G, const TIn* krow, bool valid, float* s)
{
    constexpr int E = U4<TIn>::E;
    constexpr int ROW_U4 = D / E;                    // 16-byte pieces of a row
    constexpr int CH = ROW_U4 < MaxInFlight ? ROW_U4 : MaxInFlight;
    const uint4* kr = reinterpret_cast<const uint4*>(krow);
    float2 s2[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) s2[h] = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < ROW_U4; c += CH) {
        uint4 r[CH];
#pragma unroll
        for (int u = 0; u < CH; ++u) r[u] = valid ? __ldg(kr + c + u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < CH; ++u) dot16<TIn, D, GM>(rows, G, (c + u) * E, r[u], s2);
    }
#pragma unroll
    for (int h = 0; h < GM; ++h) s[h] = s2[h].x + s2[h].y;
}

// acc[e] += w * v[e] for P (even) consecutive values, as packed fp32x2 FMAs.
template <int P>
__device__ __forceinline__ void axpy2(float w, const float* v, float* acc)
{
#pragma unroll
    for (int e = 0; e < P; e += 2) {
        const float2 r = __ffma2_rn(make_float2(w, w), make_float2(v[e], v[e + 1]), make_float2(acc[e], acc[e + 1]));
        acc[e] = r.x;
        acc[e + 1] = r.y;
    }
}

// V / K rows (dims layout) a warp loads at once: fewer when more heads'
// state is held in registers.
template <int GM> struct InFlight { static constexpr int fwd = GM <= 4 ? 16 : 8, bwd = GM <= 4 ? 8 : 4; };

// Forward: warp w of CTA x takes row 8 x + w of the (batch, kv-head, row)
// grid, for the G q-heads of the kv-head.  Keys go in batches of 32: lane j
// reads key j's whole K row and scores it against the G queries (shared
// memory); a running softmax per head (per-lane partial sums); then P V
// with lanes over the head dims, 16 V rows in flight, each key's weights
// broadcast from its lane.  GM >= G bounds the heads held in registers.
template <typename TIn, int D, int GM>
__global__ void __launch_bounds__(kThreads, GM <= 4 ? 2 : 1)
causal_fwd_kernel(const TIn* __restrict__ Q, const TIn* __restrict__ K, const TIn* __restrict__ V,
                  const int32_t* __restrict__ gidx, float* __restrict__ O, float* __restrict__ lse, int Hq, int Hkv,
                  int G, int64_t T_hist, int64_t T_seg, int64_t cap, int wg, float scale)
{
    pdl_wait();
    pdl_trigger();
    constexpr int P = D / 32;
    __shared__ __align__(16) float qsm[kWarps][GM * D];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * kWarps + warp;
    const int64_t bg = row / T_seg, i = row % T_seg;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    const int64_t pos = T_hist + i, own0 = pos / kChunk * kChunk;
    const int32_t* grow = gidx + row * wg;
    const int n_g = prefix_count(grow, wg, lane);
    const int n_keys = kGroup * n_g + int(pos - own0) + 1;
    const TIn* Kb = K + bg * cap * D;            // K / V rows of (b, g): cap apart
    const TIn* Vb = V + bg * cap * D;
    float* qw = qsm[warp];
    for (int h = 0; h < G; ++h) {
        float x[P];
        Row<TIn, P>::load(Q + ((b * Hq + g * G + h) * T_seg + i) * D + lane * P, x);
#pragma unroll
        for (int e = 0; e < P; ++e) qw[h * D + lane * P + e] = x[e];
    }
    __syncwarp();
    float m[GM], lp[GM], acc[GM][P];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        m[h] = -INFINITY;
        lp[h] = 0.f;
#pragma unroll
        for (int e = 0; e < P; ++e) acc[h][e] = 0.f;
    }
    for (int k0 = 0; k0 < n_keys; k0 += 32) {
        const bool valid = k0 + lane < n_keys;
        const int64_t t = valid ? row_token(grow, n_g, own0, k0 + lane, chk::kSiteCausalFwd) : 0;
        float s[GM], p[GM];
        row_dots<TIn, D, GM>(qw, G, Kb + t * D, valid, s);
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            if (h >= G) break;
            const float sv = valid ? s[h] * scale : -INFINITY;
            const float mn = fmaxf(m[h], warp_max(sv));
            const float c = expf(m[h] - mn);
            p[h] = expf(sv - mn);
            lp[h] = fmaf(lp[h], c, p[h]);
#pragma unroll
            for (int e = 0; e < P; ++e) acc[h][e] *= c;
            m[h] = mn;
        }
        const int nb = min(32, n_keys - k0);
        constexpr int NV = InFlight<GM>::fwd;
        for (int j0 = 0; j0 < nb; j0 += NV) {
            float vv[NV][P];
#pragma unroll
            for (int jj = 0; jj < NV; ++jj) {
                const int64_t tj = __shfl_sync(0xFFFFFFFFu, t, (j0 + jj) & 31);
                if (j0 + jj < nb) {
                    Row<TIn, P>::load(Vb + tj * D + lane * P, vv[jj]);
                } else {
#pragma unroll
                    for (int e = 0; e < P; ++e) vv[jj][e] = 0.f;
                }
            }
#pragma unroll
            for (int jj = 0; jj < NV; ++jj) {
#pragma unroll
                for (int h = 0; h < GM; ++h) {
                    if (h >= G) break;
                    const float pj = __shfl_sync(0xFFFFFFFFu, p[h], (j0 + jj) & 31);
                    axpy2<P>(pj, vv[jj], acc[h]);
                }
            }
        }
    }
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        if (h >= G) break;
        const float l = warp_sum(lp[h]);
        const int64_t orow = (b * Hq + g * G + h) * T_seg + i;
        const float inv = 1.0f / l;
#pragma unroll
        for (int e = 0; e < P; ++e) O[orow * D + lane * P + e] = acc[h][e] * inv;
        if (lane == 0) lse[orow] = m[h] + logf(l);
    }
}

// Vector float atomic add of P consecutive values (16- or 8-byte aligned).
template <int P> __device__ __forceinline__ void atomic_add_vec(float* p, const float* v);
template <> __device__ __forceinline__ void atomic_add_vec<4>(float* p, const float* v)
{
    atomicAdd(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
}
template <> __device__ __forceinline__ void atomic_add_vec<2>(float* p, const float* v)
{
    atomicAdd(reinterpret_cast<float2*>(p), make_float2(v[0], v[1]));
}

// Dynamic shared memory of the backward: per warp the G queries and the G
// output gradients of its row (floats).
__host__ __device__ inline size_t bwd_smem(int GM, int D) { return 2 * (size_t)kWarps * GM * D * sizeof(float); }

// Backward with the routing frozen.  Keys in batches of 32: lane j reads key
// j's K and V rows and forms, per head, P = exp(s - lse), dP = dO . V and
// dS = P (dP - D) with D = dO . O.  Then, lanes over the head dims (K rows
// 16 in flight), each key's dS and P broadcast from its lane: dQ += scale dS
// K in registers; the key's dK = scale sum_h dS q_h and dV = sum_h P dO_h go
// to dK_seg / dV_seg with vector atomics when it is a segment key (history
// gets no gradient).
template <typename TIn, int D, int GM>
__global__ void __launch_bounds__(kThreads, GM <= 4 ? 2 : 1)
causal_bwd_kernel(const TIn* __restrict__ Q, const TIn* __restrict__ K, const TIn* __restrict__ V,
                  const float* __restrict__ O, const float* __restrict__ lse, const TIn* __restrict__ dO,
                  const int32_t* __restrict__ gidx, float* __restrict__ dQ, float* __restrict__ dK_seg,
                  float* __restrict__ dV_seg, int Hq, int Hkv, int G, int64_t T_hist, int64_t T_seg, int64_t cap,
                  int wg, float scale)
{
    pdl_wait();
    pdl_trigger();
    constexpr int P = D / 32;
    extern __shared__ __align__(16) float bsm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * kWarps + warp;
    const int64_t bg = row / T_seg, i = row % T_seg;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    const int64_t pos = T_hist + i, own0 = pos / kChunk * kChunk;
    const int32_t* grow = gidx + row * wg;
    const int n_g = prefix_count(grow, wg, lane);
    const int n_keys = kGroup * n_g + int(pos - own0) + 1;
    const TIn* Kb = K + bg * cap * D;            // K / V rows of (b, g): cap apart
    const TIn* Vb = V + bg * cap * D;
    float* dKb = dK_seg + bg * T_seg * D + lane * P;
    float* dVb = dV_seg + bg * T_seg * D + lane * P;
    float* qw = bsm + (size_t)warp * 2 * GM * D;
    float* dow = qw + GM * D;
    float qv[GM][P], dov[GM][P], dq[GM][P], Dh[GM], lh[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        Dh[h] = 0.f;
        lh[h] = 0.f;
#pragma unroll
        for (int e = 0; e < P; ++e) qv[h][e] = dov[h][e] = dq[h][e] = 0.f;
        if (h < G) {
            const int64_t qrow = (b * Hq + g * G + h) * T_seg + i;
            Row<TIn, P>::load(Q + qrow * D + lane * P, qv[h]);
            Row<TIn, P>::load(dO + qrow * D + lane * P, dov[h]);
            float o[P];
            Row<float, P>::load(O + qrow * D + lane * P, o);
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < P; ++e) {
                a = fmaf(dov[h][e], o[e], a);
                qw[h * D + lane * P + e] = qv[h][e];
                dow[h * D + lane * P + e] = dov[h][e];
            }
            Dh[h] = warp_sum(a);
            lh[h] = __ldg(lse + qrow);
        }
    }
    __syncwarp();
    for (int k0 = 0; k0 < n_keys; k0 += 32) {
        const bool valid = k0 + lane < n_keys;
        const int64_t t = valid ? row_token(grow, n_g, own0, k0 + lane, chk::kSiteCausalBwd) : 0;
        float s[GM], dp[GM], p[GM], ds[GM];
        row_dots<TIn, D, GM, 8>(qw, G, Kb + t * D, valid, s);
        row_dots<TIn, D, GM, 8>(dow, G, Vb + t * D, valid, dp);
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            p[h] = valid && h < G ? expf(s[h] * scale - lh[h]) : 0.f;
            ds[h] = p[h] * (dp[h] - Dh[h]);
        }
        const int nb = min(32, n_keys - k0);
        constexpr int NK = InFlight<GM>::bwd;
        for (int j0 = 0; j0 < nb; j0 += NK) {
            float kv[NK][P];
            int64_t tj[NK];
#pragma unroll
            for (int jj = 0; jj < NK; ++jj) {
                tj[jj] = __shfl_sync(0xFFFFFFFFu, t, (j0 + jj) & 31);
                if (j0 + jj < nb) {
                    Row<TIn, P>::load(Kb + tj[jj] * D + lane * P, kv[jj]);
                } else {
#pragma unroll
                    for (int e = 0; e < P; ++e) kv[jj][e] = 0.f;
                }
            }
#pragma unroll
            for (int jj = 0; jj < NK; ++jj) {
                float dk[P], dv[P];
#pragma unroll
                for (int e = 0; e < P; ++e) dk[e] = dv[e] = 0.f;
#pragma unroll
                for (int h = 0; h < GM; ++h) {
                    if (h >= G) break;
                    const float dsj = scale * __shfl_sync(0xFFFFFFFFu, ds[h], (j0 + jj) & 31);
                    const float pj = __shfl_sync(0xFFFFFFFFu, p[h], (j0 + jj) & 31);
                    axpy2<P>(dsj, kv[jj], dq[h]);
                    axpy2<P>(dsj, qv[h], dk);
                    axpy2<P>(pj, dov[h], dv);
                }
                if (j0 + jj < nb && tj[jj] >= T_hist) {
                    const int64_t st = tj[jj] - T_hist;
                    atomic_add_vec<P>(dKb + st * D, dk);
                    atomic_add_vec<P>(dVb + st * D, dv);
                }
            }
        }
    }
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        if (h >= G) break;
        const int64_t qrow = (b * Hq + g * G + h) * T_seg + i;
#pragma unroll
        for (int e = 0; e < P; ++e) dQ[qrow * D + lane * P + e] = dq[h][e];
    }
}

// Shapes the window kernel takes: contexts up to 2048 chunks, k_c <= 32,
// its shared memory within a CTA's.
bool route_win_supported(const Shape& s)
{
    return s.nC <= 2048 && s.wc <= 32 && s.T_seg % rwin::kW == 0 &&
           win_layout(s.nC, s.wc, s.d).total + 1024 <= 227 * 1024;
}

template <typename TIn, int D>
cudaError_t launch_route(const Shape& s, const void* Q, const float* csum, const float* gsum, int32_t* cidx,
                         int32_t* gidx, cudaStream_t st)
{
    if (route_win_supported(s)) {
        const size_t smem = win_layout(s.nC, s.wc, D).total;
        auto k = causal_route_win_kernel<TIn, D>;
        cudaError_t e = allow_smem(k, (int)smem);
        if (e != cudaSuccess) return e;
        const unsigned grid = (unsigned)(s.B * s.Hkv * s.T_seg / rwin::kW);
        return launch_pdl(k, dim3(grid), dim3(rwin::kWinThreads), smem, st, static_cast<const TIn*>(Q), csum, gsum,
                          cidx, gidx, s.Hq, s.Hkv, s.G, s.T_hist, s.T_seg, s.cap, s.k_c, s.wc, s.k_g, s.wg);
    }
    const size_t smem = kWarps * route_warp_layout(s.nC, s.wc, D).total;
    auto k = causal_route_kernel<TIn, D>;
    cudaError_t e = allow_smem(k, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(s.B * s.Hkv * s.T_seg / kWarps);
    return launch_pdl(k, dim3(grid), dim3(kThreads), smem, st, static_cast<const TIn*>(Q), csum, gsum, cidx, gidx,
                      s.Hq, s.Hkv, s.G, s.T_hist, s.T_seg, s.cap, s.k_c, s.wc, s.k_g, s.wg);
}

template <typename TIn, int D, int GM>
cudaError_t launch_fwd(const Shape& s, const void* Q, const void* K, const void* V, const int32_t* gidx, float* O,
                       float* lse, cudaStream_t st)
{
    const unsigned grid = (unsigned)(s.B * s.Hkv * s.T_seg / kWarps);
    return launch_pdl(causal_fwd_kernel<TIn, D, GM>, dim3(grid), dim3(kThreads), 0, st, static_cast<const TIn*>(Q),
                      static_cast<const TIn*>(K), static_cast<const TIn*>(V), gidx, O, lse, s.Hq, s.Hkv, s.G,
                      s.T_hist, s.T_seg, s.cap, s.wg, s.scale);
}

template <typename TIn, int D, int GM>
cudaError_t launch_bwd(const Shape& s, const void* Q, const void* K, const void* V, const float* O, const float* lse,
                       const void* dO, const int32_t* gidx, float* dQ, float* dK, float* dV, cudaStream_t st)
{
    const size_t seg_bytes = sizeof(float) * (size_t)s.B * s.Hkv * s.T_seg * s.d;
    cudaError_t e = cudaMemsetAsync(dK, 0, seg_bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dV, 0, seg_bytes, st);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(s.B * s.Hkv * s.T_seg / kWarps);
    const size_t smem = bwd_smem(GM, D);
    auto k = causal_bwd_kernel<TIn, D, GM>;
    if ((e = allow_smem(k, (int)smem)) != cudaSuccess) return e;
    return launch_pdl(k, dim3(grid), dim3(kThreads), smem, st, static_cast<const TIn*>(Q),
                      static_cast<const TIn*>(K), static_cast<const TIn*>(V), O, lse, static_cast<const TIn*>(dO),
                      gidx, dQ, dK, dV, s.Hq, s.Hkv, s.G, s.T_hist, s.T_seg, s.cap, s.wg, s.scale);
}

// Dispatch over input type, head dim and the bound on heads per kv-head.
template <template <typename, int, int> class F, typename... A>
cudaError_t dispatch(const Shape& s, A... a)
{
    const bool small = s.G <= 4;
    if (s.dtype == HGA_BF16) {
        if (s.d == 128) return small ? F<__nv_bfloat16, 128, 4>::run(s, a...) : F<__nv_bfloat16, 128, 8>::run(s, a...);
        return small ? F<__nv_bfloat16, 64, 4>::run(s, a...) : F<__nv_bfloat16, 64, 8>::run(s, a...);
    }
    if (s.d == 128) return small ? F<float, 128, 4>::run(s, a...) : F<float, 128, 8>::run(s, a...);
    return small ? F<float, 64, 4>::run(s, a...) : F<float, 64, 8>::run(s, a...);
}

template <typename TIn, int D, int GM> struct FwdOp {
    static cudaError_t run(const Shape& s, const void* Q, const void* K, const void* V, const int32_t* gidx, float* O,
                           float* lse, cudaStream_t st)
    {
        return launch_fwd<TIn, D, GM>(s, Q, K, V, gidx, O, lse, st);
    }
};
template <typename TIn, int D, int GM> struct BwdOp {
    static cudaError_t run(const Shape& s, const void* Q, const void* K, const void* V, const float* O,
                           const float* lse, const void* dO, const int32_t* gidx, float* dQ, float* dK, float* dV,
                           cudaStream_t st)
    {
        return launch_bwd<TIn, D, GM>(s, Q, K, V, O, lse, dO, gidx, dQ, dK, dV, st);
    }
};

// ---- order of the tensor-core kernels' window items -------------------------
// The causal tensor-core kernels run one window item per CTA, and an item's
// time grows with the key tiles of its union (and, in the backward, with its
// segment tiles): 15 to 59 tiles at 16K context.  The hardware hands CTAs
// to SMs in index order as slots free up, so a heavy item drawn late ends
// well after the rest.  These two kernels order the items heaviest first
// (longest-processing-time-first list scheduling); the kernels then map
// CTA x to item order[x].
namespace csched {
constexpr int kThreads = 128;
constexpr int kMaxCost = 1023;        // costs are clamped here (they only order the items)

// Cost of the items of window u (one CTA): 2 * (union tiles + own chunk) +
// segment tiles, counted exactly as the kernels count them: the union of the
// window's rows over the groups before its own chunk, and of those the
// groups that hold segment tokens.
__global__ void __launch_bounds__(kThreads)
causal_cost_kernel(const int32_t* __restrict__ gidx, int32_t* __restrict__ cost, int64_t T_hist, int64_t T_seg,
                   int64_t nWin, int wg, int n_y)
{
    extern __shared__ uint32_t bits[];                       // bitmap of the union
    __shared__ int s_n, s_hist;
    const int64_t u = blockIdx.x, bg = u / nWin, w0 = (u % nWin) * wu::kWin;
    const int64_t limit = 8 * ((T_hist + w0) / 64);          // groups before the window's own chunk
    const int nwords = int((limit + 31) / 32);
    const int rows = int(T_seg - w0 < wu::kWin ? T_seg - w0 : wu::kWin);
    for (int w = threadIdx.x; w < nwords; w += kThreads) bits[w] = 0u;
    if (threadIdx.x == 0) {
        s_n = 0;
        s_hist = 0;
    }
    pdl_wait();
    pdl_trigger();
    __syncthreads();
    const int32_t* row0 = gidx + (bg * T_seg + w0) * wg;
    auto mark = [&](int32_t j) {
        if (j >= 0 && j < limit) atomicOr(&bits[j >> 5], 1u << (j & 31));
    };
    if ((wg & 3) == 0) {
        // The window's rows are contiguous: 16-byte loads, all issued first.
        const int n4 = rows * wg / 4;
        const int4* r4 = reinterpret_cast<const int4*>(row0);
        constexpr int kPer = 4;                              // loads in flight per thread
        for (int base = threadIdx.x; base < n4; base += kPer * kThreads) {
            int4 v[kPer];
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                const int e = base + q * kThreads;
                v[q] = e < n4 ? __ldg(r4 + e) : make_int4(-1, -1, -1, -1);
            }
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                mark(v[q].x);
                mark(v[q].y);
                mark(v[q].z);
                mark(v[q].w);
            }
        }
    } else {
        for (int e = threadIdx.x; e < rows * wg; e += kThreads) mark(__ldg(row0 + e));
    }
    __syncthreads();
    const int64_t hist_groups = T_hist / 8;                  // groups wholly in detached history
    int n = 0, h = 0;
    for (int w = threadIdx.x; w < nwords; w += kThreads) {
        const uint32_t x = bits[w];
        const int64_t lo = 32 * (int64_t)w;
        n += __popc(x);
        if (lo + 32 <= hist_groups) h += __popc(x);
        else if (lo < hist_groups) h += __popc(x & ((1u << (hist_groups - lo)) - 1u));
    }
    n = __reduce_add_sync(0xFFFFFFFFu, n);
    h = __reduce_add_sync(0xFFFFFFFFu, h);
    if ((threadIdx.x & 31) == 0) {
        atomicAdd(&s_n, n);
        atomicAdd(&s_hist, h);
    }
    __syncthreads();
    if (threadIdx.x < n_y) {
        const int nn = s_n, ch = s_hist, n_rt = (nn + 7) / 8;
        const int n_seg = ch < nn ? n_rt - ch / 8 + 1 : 1;
        const int c = 2 * (n_rt + 1) + n_seg;
        cost[u * n_y + threadIdx.x] = c < kMaxCost ? c : kMaxCost;
    }
}

// order[0 .. n) = the items by descending cost (cost[i] = order[n + i]),
// equal costs in index order.  One CTA of kMaxCost + 1 threads: the costs
// into shared memory (when they fit) with a histogram, the histogram's
// exclusive prefix from the top (thread t owns cost kMaxCost - t), then one
// warp places the items 32 at a time.
constexpr int kOrderThreads = kMaxCost + 1;
__global__ void __launch_bounds__(kOrderThreads) causal_order_kernel(int32_t* __restrict__ order, int n,
                                                                     bool keys_in_smem)
{
    extern __shared__ int32_t s_cost[];                      // [n] when keys_in_smem
    __shared__ int cursor[kMaxCost + 1];
    __shared__ int wsum[32];
    const int32_t* cost = order + n;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    cursor[threadIdx.x] = 0;
    pdl_wait();
    pdl_trigger();
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kOrderThreads) {
        int32_t c = __ldg(cost + i);
        c = c < 0 ? 0 : (c > kMaxCost ? kMaxCost : c);     // in range as written; kept in the bins regardless
        if (keys_in_smem) s_cost[i] = c;
        atomicAdd(&cursor[c], 1);
    }
    __syncthreads();
    {
        const int c = kMaxCost - int(threadIdx.x);
        const int cnt = cursor[c];
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int v = wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, v, o);
                if (lane >= o) v += y;
            }
            wsum[lane] = v;
        }
        __syncthreads();
        cursor[c] = incl - cnt + (warp ? wsum[warp - 1] : 0);   // items of higher cost
        __syncthreads();
    }
    if (warp == 0) {
        const int32_t* keys = keys_in_smem ? s_cost : cost;
        for (int base = 0; base < n; base += 32) {
            const int i = base + lane;
            int key = -1;
            if (i < n) {
                key = keys[i];
                key = key < 0 ? 0 : (key > kMaxCost ? kMaxCost : key);
            }
            const unsigned same = __match_any_sync(0xFFFFFFFFu, key);
            if (i < n) order[cursor[key] + __popc(same & ((1u << lane) - 1u))] = i;
            __syncwarp();
            if (i < n && lane == 31 - __clz(same)) cursor[key] += __popc(same);
            __syncwarp();
        }
    }
}
}  // namespace csched

}  // namespace

size_t route_causal_smem(const Shape& s)
{
    return route_win_supported(s) ? win_layout(s.nC, s.wc, s.d).total
                                  : kWarps * route_warp_layout(s.nC, s.wc, s.d).total;
}
int causal_max_heads() { return kMaxG; }

cudaError_t launch_route_causal(const Shape& s, const void* Q, const float* csum, const float* gsum, int32_t* cidx,
                                int32_t* gidx, cudaStream_t st)
{
    if (s.dtype == HGA_BF16)
        return s.d == 128 ? launch_route<__nv_bfloat16, 128>(s, Q, csum, gsum, cidx, gidx, st)
                          : launch_route<__nv_bfloat16, 64>(s, Q, csum, gsum, cidx, gidx, st);
    return s.d == 128 ? launch_route<float, 128>(s, Q, csum, gsum, cidx, gidx, st)
                      : launch_route<float, 64>(s, Q, csum, gsum, cidx, gidx, st);
}

cudaError_t launch_attn_fwd_causal(const Shape& s, const void* Q, const void* K, const void* V, const int32_t* gidx,
                                   const int32_t* sched, float* O, float* lse, cudaStream_t st)
{
    // bf16 on the tensor cores (windows of neighbouring positions over the
    // union of their routed groups); otherwise one warp per position.
    if (attn_fwd_tc_causal_supported(s)) return launch_attn_fwd_tc_causal(s, Q, K, V, gidx, sched, O, lse, st);
    return dispatch<FwdOp>(s, Q, K, V, gidx, O, lse, st);
}

cudaError_t launch_attn_bwd_causal(const Shape& s, const void* Q, const void* K, const void* V, const float* O,
                                   const float* lse, const void* dO, const int32_t* gidx, const int32_t* sched,
                                   float* dQ, float* dK, float* dV, cudaStream_t st)
{
    // bf16 on the tensor cores (the forward's windows); otherwise one warp
    // per position.
    if (attn_bwd_tc_causal_supported(s))
        return launch_attn_bwd_tc_causal(s, Q, K, V, O, lse, dO, gidx, sched, dQ, dK, dV, st);
    return dispatch<BwdOp>(s, Q, K, V, O, lse, dO, gidx, dQ, dK, dV, st);
}

int64_t causal_items(const Shape& s)
{
    return (int64_t)s.B * s.Hkv * ((s.T_seg + wu::kWin - 1) / wu::kWin) * ((s.G + 3) / 4);
}

size_t causal_sched_smem(const Shape& s) { return 4 * (size_t)((s.nG + 31) / 32); }

cudaError_t launch_causal_schedule(const Shape& s, const int32_t* gidx, int32_t* sched, cudaStream_t st)
{
    const int64_t n_win = (int64_t)s.B * s.Hkv * ((s.T_seg + wu::kWin - 1) / wu::kWin);
    const int n_y = (s.G + 3) / 4;
    const int n = (int)causal_items(s);
    if (n == 0) return cudaSuccess;
    const size_t smem = causal_sched_smem(s);
    cudaError_t e = allow_smem(csched::causal_cost_kernel, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(csched::causal_cost_kernel, dim3((unsigned)n_win), dim3(csched::kThreads), smem, st, gidx,
                   sched + n, s.T_hist, s.T_seg, (int64_t)((s.T_seg + wu::kWin - 1) / wu::kWin), s.wg, n_y);
    if (e != cudaSuccess) return e;
    // The costs in shared memory when they fit (all but huge problems).
    const size_t key_bytes = 4 * (size_t)n;
    const bool in_smem = key_bytes <= 160 * 1024;
    if (in_smem && (e = allow_smem(csched::causal_order_kernel, (int)key_bytes)) != cudaSuccess) return e;
    return launch_pdl(csched::causal_order_kernel, dim3(1), dim3(csched::kOrderThreads), in_smem ? key_bytes : 0,
                      st, sched, n, in_smem);
}

// Check word of this translation unit's bounds checks (checked builds).
HGA_CHECK_WORD_READER(check_word_causal)

}  // namespace hga
