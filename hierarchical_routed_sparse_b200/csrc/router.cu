// router.cu -- a2 + a3 block queries and chunk routing, a4 group routing.
//
// Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com),
// section "What HGA does differently": the query scores the chunk summaries
// and picks the top-k chunks, then opens those chunks at the level of
// 8-token groups and keeps the top-k groups.  Section "The one real caveat:
// causal leakage": a block's routing depends on the scores of several query
// positions -- here the block query is the mean of the block's 64 queries
// over the G q-heads sharing the kv-head.
//
// Scores are float32 dot products of float32 block queries with float32
// summaries.  Selection uses 64-bit keys (order-preserving score bits, then
// the inverted index), so "higher score, then lower index" is one unsigned
// comparison and every candidate key is distinct.
#include "hga_internal.cuh"

namespace hga {

size_t route_chunks_smem(const Shape& s);
size_t route_groups_smem(const Shape& s);

namespace {

constexpr int kRouterThreads = 256;
constexpr int kRouterWarps = kRouterThreads / 32;

// Dot product of the block query in shared memory with one summary row, by
// one warp: lane l owns elements [l*D/32, (l+1)*D/32).
template <int D>
__device__ __forceinline__ float warp_dot(const float* __restrict__ qs, const float* __restrict__ row,
                                          int lane)
{
    constexpr int P = D / 32;
    float a = 0.f;
    if constexpr (P == 4) {
        const float4 r = __ldg(reinterpret_cast<const float4*>(row) + lane);
        const float4 q = reinterpret_cast<const float4*>(qs)[lane];
        a = r.x * q.x + r.y * q.y + r.z * q.z + r.w * q.w;
    } else {
        const float2 r = __ldg(reinterpret_cast<const float2*>(row) + lane);
        const float2 q = reinterpret_cast<const float2*>(qs)[lane];
        a = r.x * q.x + r.y * q.y;
    }
    return warp_sum(a);
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

// ---- a2 + a3: one CTA per (batch, kv-head, query block) ----------------------
template <typename TIn, int D>
__global__ void __launch_bounds__(kRouterThreads)
route_chunks_kernel(const TIn* __restrict__ Q, const float* __restrict__ csum,
                    float* __restrict__ qbar, int32_t* __restrict__ cidx,
                    int Hq, int Hkv, int G, int64_t T_seg, int64_t nQB, int64_t nC,
                    int64_t c_hist, int k_c, int wc, float inv_rows)
{
    constexpr int E = Vec16<TIn>::E;
    constexpr int V16 = D / E;
    constexpr int RL = kRouterThreads / V16;          // row lanes
    extern __shared__ unsigned long long keys[];      // [nC]
    __shared__ float part[RL][D];
    __shared__ __align__(16) float qs[D];

    const int64_t u = blockIdx.x;                      // ((b*Hkv)+g)*nQB + qb
    const int64_t qb = u % nQB, bg = u / nQB;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // a2: block query = mean over G heads x 64 queries.
    {
        const int v = tid % V16, rl = tid / V16;
        float acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.f;
        for (int r = rl; r < G * kChunk; r += RL) {
            const int64_t h = g * G + r / kChunk;
            const TIn* src = Q + ((b * Hq + h) * T_seg + qb * kChunk + r % kChunk) * D + v * E;
            float x[E];
            Vec16<TIn>::load(src, x);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += x[e];
        }
#pragma unroll
        for (int e = 0; e < E; ++e) part[rl][v * E + e] = acc[e];
    }
    __syncthreads();
    for (int col = tid; col < D; col += kRouterThreads) {
        float a = 0.f;
#pragma unroll 8
        for (int r = 0; r < RL; ++r) a += part[r][col];
        a *= inv_rows;
        qs[col] = a;
        qbar[u * D + col] = a;
    }
    __syncthreads();

    // a3: scores of the eligible chunks c < c0 (strictly before the own chunk).
    const int c0 = static_cast<int>(c_hist + qb);
    int32_t* out = cidx + u * wc;
    if (k_c <= 0 || k_c >= c0) {                       // keep every eligible chunk
        for (int i = tid; i < wc; i += kRouterThreads) out[i] = i < c0 ? i : -1;
        return;
    }
    const float* cs = csum + bg * nC * D;
    for (int c = warp; c < c0; c += kRouterWarps) {
        const float sc = warp_dot<D>(qs, cs + (int64_t)c * D, lane);
        if (lane == 0) keys[c] = pack_key(sc, c);
    }
    __syncthreads();
    if (warp != 0) return;
    // Warp-level top-k: k rounds of a warp arg-max; the winner's key is
    // cleared to 0, which marks it selected.
    for (int round = 0; round < k_c; ++round) {
        unsigned long long best = 0ull;
        for (int c = lane; c < c0; c += 32) best = keys[c] > best ? keys[c] : best;
        best = warp_max_u64(best);
        __syncwarp();
        if (lane == 0) keys[key_index(best)] = 0ull;
        __syncwarp();
    }
    compact_selected(keys, nullptr, c0, out, wc, lane);
}

// ---- a4: one CTA per (batch, kv-head, query block) ---------------------------
template <int D>
__global__ void __launch_bounds__(kRouterThreads)
route_groups_kernel(const float* __restrict__ qbar, const float* __restrict__ gsum,
                    const int32_t* __restrict__ cidx, int32_t* __restrict__ gidx,
                    int64_t nQB, int64_t nG, int wc, int k_g, int wg)
{
    extern __shared__ unsigned long long keys[];      // [8*wc], ids [8*wc], flags [8*wc]
    int32_t* ids = reinterpret_cast<int32_t*>(keys + (size_t)kGroupsPerChunk * wc);
    uint8_t* flags = reinterpret_cast<uint8_t*>(ids + (size_t)kGroupsPerChunk * wc);
    __shared__ __align__(16) float qs[D];
    __shared__ int n_valid;

    const int64_t u = blockIdx.x;
    const int64_t bg = u / nQB;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t* crow = cidx + u * wc;

    for (int col = tid; col < D; col += kRouterThreads) qs[col] = qbar[u * D + col];
    if (warp == 0) {                                   // valid chunks form a prefix
        int n = 0;
        for (int base = 0; base < wc; base += 32) {
            const int i = base + lane;
            n += __popc(__ballot_sync(0xFFFFFFFFu, i < wc && crow[i] >= 0));
        }
        if (lane == 0) n_valid = n;
    }
    __syncthreads();
    const int n = n_valid * kGroupsPerChunk;           // candidate groups
    for (int i = tid; i < n; i += kRouterThreads)
        ids[i] = crow[i / kGroupsPerChunk] * kGroupsPerChunk + i % kGroupsPerChunk;
    int32_t* out = gidx + u * wg;
    __syncthreads();
    if (k_g <= 0 || k_g >= n) {                        // keep every candidate
        for (int i = tid; i < wg; i += kRouterThreads) out[i] = i < n ? ids[i] : -1;
        return;
    }
    const float* gs = gsum + bg * nG * D;
    for (int i = warp; i < n; i += kRouterWarps) {
        const float sc = warp_dot<D>(qs, gs + (int64_t)ids[i] * D, lane);
        if (lane == 0) keys[i] = pack_key(sc, ids[i]);
    }
    __syncthreads();
    // Rank selection: a candidate is kept when fewer than k_g keys beat it.
    // Flags are gathered first, then written as key 0 for the compaction.
    for (int i = tid; i < n; i += kRouterThreads) {
        const unsigned long long ki = keys[i];
        int rank = 0;
        for (int j = 0; j < n; ++j) rank += keys[j] > ki;
        flags[i] = rank < k_g;
    }
    __syncthreads();
    for (int i = tid; i < n; i += kRouterThreads)
        if (flags[i]) keys[i] = 0ull;
    __syncthreads();
    if (warp == 0) compact_selected(keys, ids, n, out, wg, lane);
}

template <typename TIn, int D>
cudaError_t launch_rc(const Shape& s, const void* Q, const float* csum, float* qbar, int32_t* cidx,
                      cudaStream_t st)
{
    const size_t smem = route_chunks_smem(s);
    auto k = route_chunks_kernel<TIn, D>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t blocks = (int64_t)s.B * s.Hkv * s.nQB;
    k<<<(unsigned)blocks, kRouterThreads, smem, st>>>(
        static_cast<const TIn*>(Q), csum, qbar, cidx, s.Hq, s.Hkv, s.G, s.T_seg, s.nQB, s.nC,
        s.T_hist / kChunk, s.k_c, s.wc, 1.0f / (float)(s.G * kChunk));
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_rg(const Shape& s, const float* qbar, const float* gsum, const int32_t* cidx,
                      int32_t* gidx, cudaStream_t st)
{
    const size_t smem = route_groups_smem(s);
    auto k = route_groups_kernel<D>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t blocks = (int64_t)s.B * s.Hkv * s.nQB;
    k<<<(unsigned)blocks, kRouterThreads, smem, st>>>(qbar, gsum, cidx, gidx, s.nQB, s.nG, s.wc,
                                                      s.k_g, s.wg);
    return cudaGetLastError();
}

}  // namespace

size_t route_chunks_smem(const Shape& s) { return sizeof(unsigned long long) * (size_t)s.nC; }
size_t route_groups_smem(const Shape& s)
{
    return (sizeof(unsigned long long) + sizeof(int32_t) + 1) * kGroupsPerChunk * (size_t)s.wc;
}

cudaError_t launch_route_chunks(const Shape& s, const void* Q, const float* csum, float* qbar,
                                int32_t* cidx, cudaStream_t st)
{
    if (s.dtype == HGA_BF16)
        return s.d == 128 ? launch_rc<__nv_bfloat16, 128>(s, Q, csum, qbar, cidx, st)
                          : launch_rc<__nv_bfloat16, 64>(s, Q, csum, qbar, cidx, st);
    return s.d == 128 ? launch_rc<float, 128>(s, Q, csum, qbar, cidx, st)
                      : launch_rc<float, 64>(s, Q, csum, qbar, cidx, st);
}

cudaError_t launch_route_groups(const Shape& s, const float* qbar, const float* gsum,
                                const int32_t* cidx, int32_t* gidx, cudaStream_t st)
{
    return s.d == 128 ? launch_rg<128>(s, qbar, gsum, cidx, gidx, st)
                      : launch_rg<64>(s, qbar, gsum, cidx, gidx, st);
}

}  // namespace hga
