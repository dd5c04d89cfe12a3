// router_core.cuh -- device pieces of the routing (a3, a4) shared by the
// segment router (router.cu) and the decode step (decode.cu): candidate
// scoring, warp-level top-k and the chunk / group selection of one block.
//
// Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com),
// section "What HGA does differently": the block query scores the chunk
// summaries and keeps the top-k chunks, then the top-k groups of those
// chunks.  Selection uses 64-bit keys (order-preserving score bits, then the
// inverted index), so "higher score, then lower index" is one unsigned
// comparison and every candidate key is distinct.  Not part of the ABI.
#pragma once

#include <stdint.h>

#include "check.cuh"

#include "hga_internal.cuh"

namespace hga {
namespace rt {

constexpr int kRouterThreads = 256;
constexpr int kRouterWarps = kRouterThreads / 32;
constexpr int kBatch = 16;          // candidates a warp scores at once

// The barrier of the per-block routing pieces below, which run on
// kRouterThreads threads: the CTA barrier by default; a kernel whose CTA has
// more threads (the fused route + forward kernel) runs them on its first
// kRouterThreads threads with a named barrier over those.
struct SyncCta {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
struct SyncRouterThreads {
    __device__ __forceinline__ void operator()() const
    {
        asm volatile("bar.sync 1, %0;" ::"n"(kRouterThreads) : "memory");
    }
};

// Scores of candidates 0..n-1 against the block query qs (shared memory):
// score(c) = qs . row(c), written as a selection key into keys[c].  Warp w
// of `Warps` takes batches of 16 candidates w, w+Warps, ...; for each batch every lane
// issues its 16 coalesced loads (lane l holds elements [l*P, (l+1)*P) of each
// row) before any arithmetic, so a batch costs one memory round trip, and
// the 16 partial sums are reduced across the warp with 16 shuffles (each
// step halves the values a lane carries).
template <int D, int Warps = kRouterWarps, typename RowFn>
__device__ __forceinline__ void score_candidates(const float* __restrict__ qs, int n, RowFn row_of,
                                                 unsigned long long* keys, int warp, int lane)
{
    constexpr int P = D / 32;
    float q[P];
#pragma unroll
    for (int e = 0; e < P; ++e) q[e] = qs[lane * P + e];
    for (int base = warp * kBatch; base < n; base += Warps * kBatch) {
        float v[kBatch];
        int32_t id[kBatch];
        float x[kBatch][P];
#pragma unroll
        for (int c = 0; c < kBatch; ++c) {
            const int cc = base + c < n ? base + c : base;
            const float* row;
            id[c] = row_of(cc, row);
            if constexpr (P == 4) {
                const float4 t = __ldg(reinterpret_cast<const float4*>(row) + lane);
                x[c][0] = t.x; x[c][1] = t.y; x[c][2] = t.z; x[c][3] = t.w;
            } else {
                const float2 t = __ldg(reinterpret_cast<const float2*>(row) + lane);
                x[c][0] = t.x; x[c][1] = t.y;
            }
        }
#pragma unroll
        for (int c = 0; c < kBatch; ++c) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < P; ++e) a = fmaf(x[c][e], q[e], a);
            v[c] = a;
        }
        // Transpose-reduce: after the step with offset o the lane keeps the
        // half of its values selected by its lane bit o.
#pragma unroll
        for (int o = 16, m = kBatch / 2; o >= 2; o >>= 1, m >>= 1) {
            const bool up = lane & o;
#pragma unroll
            for (int c = 0; c < m; ++c) {
                const float send = up ? v[c] : v[c + m];
                const float keep = up ? v[c + m] : v[c];
                v[c] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
            }
        }
        v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], 1);
        // Lane l now holds the full score of candidate ((l >> 1) & 15) in
        // bit order 16, 8, 4, 2 -> 8, 4, 2, 1.
        const int c = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
        int32_t my_id = id[0];
#pragma unroll
        for (int k = 1; k < kBatch; ++k) my_id = c == k ? id[k] : my_id;
        if ((lane & 1) == 0 && base + c < n) keys[base + c] = pack_key(v[0], my_id);
    }
}

// Write the selected candidates (key == 0 marks a selected slot) in
// ascending candidate order, then -1 up to the row width.  One warp.
__device__ __forceinline__ void compact_selected(const unsigned long long* keys, const int32_t* ids,
                                                 int n, int32_t* out, int width, int lane)
{
    int pos = 0;
    for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        const bool sel = i < n && keys[i] == 0ull;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) out[pos + __popc(m & ((1u << lane) - 1u))] = ids ? ids[i] : i;
        pos += __popc(m);
    }
    for (int i = pos + lane; i < width; i += 32) out[i] = -1;
}

// Warp-level top-k over candidate keys held in registers: lane l holds the
// keys of candidates l + 32 m (m < kRegCand; 0 = none).  A round takes the
// warp maximum with two 32-bit reductions (score bits, then the inverted
// index among equal scores); the winning lane marks its candidate (bit m of
// sel) and recomputes its maximum from registers.  Then the selected
// candidates are written in ascending candidate order, -1 up to `width`,
// to out0 and (if not null) out1.
constexpr int kRegCand = 8;

__device__ __forceinline__ void warp_topk_regs(unsigned long long (&ck)[kRegCand], int k, int32_t* out0,
                                               int32_t* out1, int width, int lane)
{
    auto lane_max = [&]() {
        unsigned long long b = ck[0];
#pragma unroll
        for (int m = 1; m < kRegCand; ++m) b = ck[m] > b ? ck[m] : b;
        return b;
    };
    unsigned long long best = lane_max();
    uint32_t sel = 0;
    for (int round = 0; round < k; ++round) {
        const uint32_t hi = uint32_t(best >> 32), lo = uint32_t(best);
        const uint32_t mhi = __reduce_max_sync(0xFFFFFFFFu, hi);
        const uint32_t mlo = __reduce_max_sync(0xFFFFFFFFu, hi == mhi ? lo : 0u);
        if (best != 0ull && hi == mhi && lo == mlo) {       // keys are distinct: one lane wins
#pragma unroll
            for (int m = 0; m < kRegCand; ++m)
                if (ck[m] == best) {
                    ck[m] = 0ull;
                    sel |= 1u << m;
                }
            best = lane_max();
        }
    }
    const unsigned below = (1u << lane) - 1u;
    int pos = 0;
#pragma unroll
    for (int m = 0; m < kRegCand; ++m) {
        const bool mine = (sel >> m) & 1u;
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, mine);
        if (mine) {
            const int at = pos + __popc(bal & below);
            out0[at] = lane + 32 * m;
            if (out1) out1[at] = lane + 32 * m;
        }
        pos += __popc(bal);
    }
    for (int i = pos + lane; i < width; i += 32) {
        out0[i] = -1;
        if (out1) out1[i] = -1;
    }
}

// a3 selection: the top-k_c of the chunk keys keys[0..c0) (all scored, block
// synchronised) on warp 0 -- from registers (warp_topk_regs) when c0 <= 256,
// else by rounds over shared memory: lane l keeps the largest key among its
// candidates l, l+32, ...; a round takes the warp maximum as above and the
// winning lane clears the winner's key (0 marks it selected) and rescans its
// candidates.  Writes the row to out0 and (if not null) out1.  Other warps
// return at once.
__device__ __forceinline__ void select_chunks(unsigned long long* keys, int c0, int k_c, int wc, int32_t* out0,
                                              int32_t* out1, int warp, int lane)
{
    if (warp != 0) return;
    if (c0 <= 32 * kRegCand) {
        unsigned long long ck[kRegCand];
#pragma unroll
        for (int m = 0; m < kRegCand; ++m) ck[m] = lane + 32 * m < c0 ? keys[lane + 32 * m] : 0ull;
        warp_topk_regs(ck, k_c, out0, out1, wc, lane);
        return;
    }
    unsigned long long best = 0ull;
    for (int c = lane; c < c0; c += 32) best = keys[c] > best ? keys[c] : best;
    for (int round = 0; round < k_c; ++round) {
        const uint32_t hi = uint32_t(best >> 32), lo = uint32_t(best);
        const uint32_t mhi = __reduce_max_sync(0xFFFFFFFFu, hi);
        const uint32_t mlo = __reduce_max_sync(0xFFFFFFFFu, hi == mhi ? lo : 0u);
        if (best != 0ull && hi == mhi && lo == mlo) {   // keys are distinct: one lane wins
            keys[key_index(best)] = 0ull;
            best = 0ull;
            for (int c = lane; c < c0; c += 32) best = keys[c] > best ? keys[c] : best;
        }
    }
    __syncwarp();
    compact_selected(keys, nullptr, c0, out0, wc, lane);
    if (out1) compact_selected(keys, nullptr, c0, out1, wc, lane);
}

// 16 bytes of inputs widened to float32 (8 bf16 or 4 float).
template <typename T> __device__ __forceinline__ void widen16(const uint4 r, float* out);
template <> __device__ __forceinline__ void widen16<__nv_bfloat16>(const uint4 r, float* out)
{
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        out[2 * i] = __uint_as_float(w[i] << 16);
        out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
template <> __device__ __forceinline__ void widen16<float>(const uint4 r, float* out)
{
    out[0] = __uint_as_float(r.x); out[1] = __uint_as_float(r.y);
    out[2] = __uint_as_float(r.z); out[3] = __uint_as_float(r.w);
}

// Block query into qs (and qbar[u]): the mean of the block's 64 queries over
// the G q-heads of the kv-head.  Every thread owns one 16-byte column vector
// and issues the loads of up to 16 of its rows (kept as raw 16-byte words)
// before widening and adding them: one memory round trip for G = 4.
template <typename TIn, int D, typename Sync = SyncCta>
__device__ __forceinline__ void block_query(const TIn* __restrict__ Q, float* __restrict__ qbar_row,
                                            float* qs, float (*part)[D], int64_t b, int64_t g, int64_t qb,
                                            int Hq, int G, int64_t T_seg, float inv_rows, int tid)
{
    const Sync sync{};
    constexpr int E = Vec16<TIn>::E;
    constexpr int V16 = D / E;
    constexpr int RL = kRouterThreads / V16;          // row lanes
    const int v = tid % V16, rl = tid / V16;
    const int rows = G * kChunk;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    constexpr int kLoads = 16;
    for (int r0 = rl; r0 < rows; r0 += kLoads * RL) {
        uint4 raw[kLoads];
#pragma unroll
        for (int q = 0; q < kLoads; ++q) {
            const int r = r0 + q * RL;
            if (r < rows) {
                const int64_t h = (int64_t)g * G + r / kChunk;
                raw[q] = __ldg(reinterpret_cast<const uint4*>(
                    Q + ((b * Hq + h) * T_seg + qb * kChunk + r % kChunk) * D + v * E));
            } else {
                raw[q] = make_uint4(0u, 0u, 0u, 0u);        // zero bits widen to 0.0f
            }
        }
#pragma unroll
        for (int q = 0; q < kLoads; ++q) {
            float x[E];
            widen16<TIn>(raw[q], x);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += x[e];
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) part[rl][v * E + e] = acc[e];
    sync();
    for (int col = tid; col < D; col += kRouterThreads) {
        float a = 0.f;
#pragma unroll 8
        for (int r = 0; r < RL; ++r) a += part[r][col];
        a *= inv_rows;
        qs[col] = a;
        qbar_row[col] = a;
    }
    sync();
}

// a3: chunk routing of one block: scores of the eligible chunks c < c0, then
// select_chunks.  Writes the row to cidx_row and (if not null) to crow_smem.
template <int D, typename Sync = SyncCta>
__device__ __forceinline__ void route_chunks_block(const float* qs, const float* __restrict__ cs, int c0, int k_c,
                                                   int wc, unsigned long long* keys, int32_t* cidx_row,
                                                   int32_t* crow_smem, int tid)
{
    const Sync sync{};
    const int lane = tid & 31, warp = tid >> 5;
    if (k_c <= 0 || k_c >= c0) {                       // keep every eligible chunk
        for (int i = tid; i < wc; i += kRouterThreads) {
            const int32_t v = i < c0 ? i : -1;
            cidx_row[i] = v;
            if (crow_smem) crow_smem[i] = v;
        }
        sync();
        return;
    }
    score_candidates<D>(qs, c0, [&](int c, const float*& row) { row = cs + (int64_t)c * D; return c; }, keys,
                        warp, lane);
    sync();
    select_chunks(keys, c0, k_c, wc, cidx_row, crow_smem, warp, lane);
    sync();
}

// Number of valid entries of an index row (an ascending prefix); one warp.
__device__ __forceinline__ int prefix_count(const int32_t* row, int w, int lane)
{
    int n = 0;
    for (int base = 0; base < w; base += 32) {
        const int i = base + lane;
        n += __popc(__ballot_sync(0xFFFFFFFFu, i < w && row[i] >= 0));
    }
    return n;
}

// a4 selection: of the n scored group candidates (keys, ids; block
// synchronised) a candidate is kept when fewer than k_g candidates beat it;
// the kept ids are written in candidate order to gidx_row.
template <typename Sync = SyncCta>
__device__ __forceinline__ void select_groups(unsigned long long* keys, const int32_t* ids, int n, int k_g,
                                              uint8_t* flags, int32_t* gidx_row, int wg, int tid)
{
    const Sync sync{};
    const int lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < n; i += kRouterThreads) {
        const unsigned long long ki = keys[i];
        int rank = 0;
        for (int j = 0; j < n; ++j) rank += keys[j] > ki;
        flags[i] = rank < k_g;
    }
    sync();
    for (int i = tid; i < n; i += kRouterThreads)
        if (flags[i]) keys[i] = 0ull;
    sync();
    if (warp == 0) compact_selected(keys, ids, n, gidx_row, wg, lane);
}

// a4: group routing of one block: the 8 groups of every chunk in crow (an
// ascending prefix of valid chunks), scored and ranked (select_groups).
template <int D, typename Sync = SyncCta>
__device__ __forceinline__ void route_groups_block(const float* qs, const float* __restrict__ gs,
                                                   const int32_t* crow, int wc, int k_g, int wg,
                                                   unsigned long long* keys, int32_t* ids, uint8_t* flags,
                                                   int* s_count, int32_t* gidx_row, int tid,
                                                   int64_t c_limit = INT64_MAX)
{
    const Sync sync{};
    const int lane = tid & 31, warp = tid >> 5;
    if (warp == 0) {
        const int n = prefix_count(crow, wc, lane);
        if (lane == 0) *s_count = n;
    }
    sync();
    const int n = *s_count * kGroupsPerChunk;          // candidate groups
    for (int i = tid; i < n; i += kRouterThreads)
        ids[i] = chk::chunk(crow[i / kGroupsPerChunk], c_limit, chk::kSiteRouteGroups) * kGroupsPerChunk +
                 i % kGroupsPerChunk;
    sync();
    if (k_g <= 0 || k_g >= n) {                        // keep every candidate
        for (int i = tid; i < wg; i += kRouterThreads) gidx_row[i] = i < n ? ids[i] : -1;
        return;
    }
    score_candidates<D>(qs, n, [&](int c, const float*& row) { row = gs + (int64_t)ids[c] * D; return ids[c]; },
                        keys, warp, lane);
    sync();
    select_groups<Sync>(keys, ids, n, k_g, flags, gidx_row, wg, tid);
}

}  // namespace rt
}  // namespace hga
