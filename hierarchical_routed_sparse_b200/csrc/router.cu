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
#include "router_core.cuh"

namespace hga {

size_t route_chunks_smem(const Shape& s);
size_t route_groups_smem(const Shape& s);
size_t route_fused_smem(const Shape& s);

namespace {

using namespace rt;

// ---- a2 + a3: one CTA per (batch, kv-head, query block) ----------------------
template <typename TIn, int D>
__global__ void __launch_bounds__(kRouterThreads, 2)
route_chunks_kernel(const TIn* __restrict__ Q, const float* __restrict__ csum,
                    float* __restrict__ qbar, int32_t* __restrict__ cidx,
                    int Hq, int Hkv, int G, int64_t T_seg, int64_t nQB, int64_t nCs,
                    int64_t c_hist, int k_c, int wc, float inv_rows)
{
    constexpr int RL = kRouterThreads / (D / Vec16<TIn>::E);
    extern __shared__ unsigned long long keys[];      // [nC]
    __shared__ float part[RL][D];
    __shared__ __align__(16) float qs[D];
    pdl_wait();
    pdl_trigger();
    const int64_t u = blockIdx.x;                      // ((b*Hkv)+g)*nQB + qb
    const int64_t qb = u % nQB, bg = u / nQB;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    block_query<TIn, D>(Q, qbar + u * D, qs, part, b, g, qb, Hq, G, T_seg, inv_rows, threadIdx.x);
    route_chunks_block<D>(qs, csum + bg * nCs * D, static_cast<int>(c_hist + qb), k_c, wc, keys, cidx + u * wc,
                          nullptr, threadIdx.x);
}

// ---- a4: one CTA per (batch, kv-head, query block) ---------------------------
template <int D>
__global__ void __launch_bounds__(kRouterThreads, 2)
route_groups_kernel(const float* __restrict__ qbar, const float* __restrict__ gsum,
                    const int32_t* __restrict__ cidx, int32_t* __restrict__ gidx,
                    int64_t nQB, int64_t nGs, int wc, int k_g, int wg, int64_t c_hist)
{
    extern __shared__ unsigned long long keys[];      // [8*wc], ids [8*wc], flags [8*wc]
    int32_t* ids = reinterpret_cast<int32_t*>(keys + (size_t)kGroupsPerChunk * wc);
    uint8_t* flags = reinterpret_cast<uint8_t*>(ids + (size_t)kGroupsPerChunk * wc);
    __shared__ __align__(16) float qs[D];
    __shared__ int n_valid;
    pdl_wait();
    pdl_trigger();
    const int64_t u = blockIdx.x;
    const int64_t bg = u / nQB;
    for (int col = threadIdx.x; col < D; col += kRouterThreads) qs[col] = qbar[u * D + col];
    __syncthreads();
    // The caller's chunk row: valid chunks lie before the block's own chunk.
    route_groups_block<D>(qs, gsum + bg * nGs * D, cidx + u * wc, wc, k_g, wg, keys, ids, flags, &n_valid,
                          gidx + u * wg, threadIdx.x, c_hist + u % nQB);
}

// ---- a2 + a3 + a4 in one launch ------------------------------------------------
template <typename TIn, int D>
__global__ void __launch_bounds__(kRouterThreads, 2)
route_fused_kernel(const TIn* __restrict__ Q, const float* __restrict__ csum, const float* __restrict__ gsum,
                   float* __restrict__ qbar, int32_t* __restrict__ cidx, int32_t* __restrict__ gidx,
                   int Hq, int Hkv, int G, int64_t T_seg, int64_t nQB, int64_t nC, int64_t nCs, int64_t nGs,
                   int64_t c_hist, int k_c, int wc, int k_g, int wg, float inv_rows)
{
    constexpr int RL = kRouterThreads / (D / Vec16<TIn>::E);
    // keys [max(nC, 8*wc)], ids [8*wc], flags [8*wc], crow [wc]
    extern __shared__ unsigned long long keys[];
    const size_t nk = (size_t)(nC > kGroupsPerChunk * wc ? nC : kGroupsPerChunk * wc);
    int32_t* ids = reinterpret_cast<int32_t*>(keys + nk);
    int32_t* crow = ids + (size_t)kGroupsPerChunk * wc;
    uint8_t* flags = reinterpret_cast<uint8_t*>(crow + wc);
    __shared__ float part[RL][D];
    __shared__ __align__(16) float qs[D];
    __shared__ int n_valid;
    pdl_wait();
    pdl_trigger();
    const int64_t u = blockIdx.x;
    const int64_t qb = u % nQB, bg = u / nQB;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    block_query<TIn, D>(Q, qbar + u * D, qs, part, b, g, qb, Hq, G, T_seg, inv_rows, threadIdx.x);
    route_chunks_block<D>(qs, csum + bg * nCs * D, static_cast<int>(c_hist + qb), k_c, wc, keys, cidx + u * wc,
                          crow, threadIdx.x);
    route_groups_block<D>(qs, gsum + bg * nGs * D, crow, wc, k_g, wg, keys, ids, flags, &n_valid, gidx + u * wg,
                          threadIdx.x);
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
    return launch_pdl(k, dim3((unsigned)blocks), dim3(kRouterThreads), smem, st, static_cast<const TIn*>(Q), csum,
                      qbar, cidx, s.Hq, s.Hkv, s.G, s.T_seg, s.nQB, s.nCs, s.T_hist / kChunk, s.k_c, s.wc,
                      1.0f / (float)(s.G * kChunk));
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
    return launch_pdl(k, dim3((unsigned)blocks), dim3(kRouterThreads), smem, st, qbar, gsum, cidx, gidx, s.nQB,
                      s.nGs, s.wc, s.k_g, s.wg, s.T_hist / kChunk);
}

template <typename TIn, int D>
cudaError_t launch_rf(const Shape& s, const void* Q, const float* csum, const float* gsum, float* qbar,
                      int32_t* cidx, int32_t* gidx, cudaStream_t st)
{
    const size_t smem = route_fused_smem(s);
    auto k = route_fused_kernel<TIn, D>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t blocks = (int64_t)s.B * s.Hkv * s.nQB;
    return launch_pdl(k, dim3((unsigned)blocks), dim3(kRouterThreads), smem, st, static_cast<const TIn*>(Q), csum,
                      gsum, qbar, cidx, gidx, s.Hq, s.Hkv, s.G, s.T_seg, s.nQB, s.nC, s.nCs, s.nGs,
                      s.T_hist / kChunk, s.k_c, s.wc, s.k_g, s.wg, 1.0f / (float)(s.G * kChunk));
}

}  // namespace

size_t route_fused_smem(const Shape& s)
{
    const size_t nk = (size_t)(s.nC > kGroupsPerChunk * (int64_t)s.wc ? s.nC : kGroupsPerChunk * (int64_t)s.wc);
    return sizeof(unsigned long long) * nk + (sizeof(int32_t) + 1) * kGroupsPerChunk * (size_t)s.wc +
           sizeof(int32_t) * (size_t)s.wc;
}

cudaError_t launch_route_fused(const Shape& s, const void* Q, const float* csum, const float* gsum, float* qbar,
                               int32_t* cidx, int32_t* gidx, cudaStream_t st)
{
    if (s.dtype == HGA_BF16)
        return s.d == 128 ? launch_rf<__nv_bfloat16, 128>(s, Q, csum, gsum, qbar, cidx, gidx, st)
                          : launch_rf<__nv_bfloat16, 64>(s, Q, csum, gsum, qbar, cidx, gidx, st);
    return s.d == 128 ? launch_rf<float, 128>(s, Q, csum, gsum, qbar, cidx, gidx, st)
                      : launch_rf<float, 64>(s, Q, csum, gsum, qbar, cidx, gidx, st);
}

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

// Check word of this translation unit's bounds checks (checked builds).
HGA_CHECK_WORD_READER(check_word_router)

}  // namespace hga
