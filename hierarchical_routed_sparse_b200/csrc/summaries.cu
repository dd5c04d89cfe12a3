// summaries.cu -- a1: chunk and group summaries of the keys.
//
// Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com),
// section "What HGA does differently": compact summary vectors of each
// 64-token chunk stay in device memory, and chunks are opened at the level
// of 8-token groups.  A summary is read as the arithmetic mean of its keys.
//
// One CTA summarises one chunk of one (batch, kv-head): 64 rows x d of K
// (16 KiB in bf16 at d = 128).  Thread (r, v) owns 16-byte column vector v
// of group r and issues its 8 row loads back to back, so every byte of K is
// read exactly once with fully coalesced 16-byte loads; the group sums
// become the group means and, summed through shared memory, the chunk mean.
// The kernel is HBM-bound: per chunk it reads 64*d input elements and
// writes 9*d floats.
#include "hga_internal.cuh"

namespace hga {
namespace {

template <typename TIn, int D>
__global__ void __launch_bounds__(kGroupsPerChunk * D / Vec16<TIn>::E)
summaries_kernel(const TIn* __restrict__ K, int64_t nCs, int64_t nGs, int64_t T_src, int64_t row0,
                 int64_t c_begin, int64_t n_chunks, float* __restrict__ csum, float* __restrict__ gsum)
{
    constexpr int E = Vec16<TIn>::E;
    constexpr int V16 = D / E;                  // 16-byte vectors per row
    __shared__ float part[kGroupsPerChunk][D];

    pdl_wait();
    pdl_trigger();
    const int64_t bg = blockIdx.x / n_chunks;   // (batch, kv-head)
    const int64_t c = c_begin + blockIdx.x % n_chunks;
    const int r = threadIdx.x / V16, v = threadIdx.x % V16;

    // K holds T_src rows per (batch, kv-head), the first at position row0.
    const TIn* src = K + (bg * T_src + c * kChunk - row0 + r * kGroup) * D + v * E;
    float x[kGroup][E];
#pragma unroll
    for (int t = 0; t < kGroup; ++t) Vec16<TIn>::load(src + t * D, x[t]);
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        float a = 0.f;
#pragma unroll
        for (int t = 0; t < kGroup; ++t) a += x[t][e];
        acc[e] = a;
    }
    float* gdst = gsum + (bg * nGs + c * kGroupsPerChunk + r) * D + v * E;
#pragma unroll
    for (int e = 0; e < E; e += 4)
        *reinterpret_cast<float4*>(gdst + e) =
            make_float4(acc[e] * 0.125f, acc[e + 1] * 0.125f, acc[e + 2] * 0.125f, acc[e + 3] * 0.125f);
#pragma unroll
    for (int e = 0; e < E; ++e) part[r][v * E + e] = acc[e];
    __syncthreads();
    for (int col = threadIdx.x; col < D; col += blockDim.x) {
        float a = 0.f;
#pragma unroll
        for (int q = 0; q < kGroupsPerChunk; ++q) a += part[q][col];
        csum[(bg * nCs + c) * D + col] = a * (1.0f / kChunk);
    }
}

template <typename TIn, int D>
cudaError_t launch(const Shape& s, const void* K, int64_t T_src, int64_t row0, int64_t c_begin, int64_t c_end,
                   float* csum, float* gsum, cudaStream_t st)
{
    const int64_t n = c_end - c_begin;
    const int64_t blocks = n * s.B * s.Hkv;
    constexpr int threads = kGroupsPerChunk * D / Vec16<TIn>::E;
    return launch_pdl(summaries_kernel<TIn, D>, dim3((unsigned)blocks), dim3(threads), 0, st,
                      static_cast<const TIn*>(K), s.nCs, s.nGs, T_src, row0, c_begin, n, csum, gsum);
}

}  // namespace

cudaError_t launch_summaries(const Shape& s, const void* K, int64_t T_src, int64_t row0, int64_t c_begin,
                             int64_t c_end, float* csum, float* gsum, cudaStream_t st)
{
    if (s.dtype == HGA_BF16)
        return s.d == 128 ? launch<__nv_bfloat16, 128>(s, K, T_src, row0, c_begin, c_end, csum, gsum, st)
                          : launch<__nv_bfloat16, 64>(s, K, T_src, row0, c_begin, c_end, csum, gsum, st);
    return s.d == 128 ? launch<float, 128>(s, K, T_src, row0, c_begin, c_end, csum, gsum, st)
                      : launch<float, 64>(s, K, T_src, row0, c_begin, c_end, csum, gsum, st);
}

}  // namespace hga
