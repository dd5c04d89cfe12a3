// decode.cu -- one generation step: the new token is a query block of one.
//
// Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com),
// section "Retrieval: no degradation in the dense baseline": HGA itself can
// also do generation.  The step follows the segment path with a block of
// one query (section "What HGA does differently"): the block query is the
// token's query averaged over the G q-heads of its kv-head; the complete
// chunks before the token's own chunk are scored against their summaries and
// the top-k_c kept; the top-k_g groups of those chunks are kept; the token
// attends the routed groups' exact tokens and its own chunk up to itself.
// A chunk's summaries exist once the chunk is complete (the caller appends
// them with hga_build_summaries as decoding fills it).
//
// One CTA per (batch, kv-head), 256 threads: routing with the segment
// router's pieces, then the G heads' scores (keys spread over the 8 warps,
// four rows in flight per warp), a softmax per head and O = P V with a
// cross-warp reduction in shared memory.  Float32 arithmetic throughout.
#include "hga_internal.cuh"
#include "router_core.cuh"

namespace hga {
namespace {

using namespace rt;

constexpr int kMaxG = 8;            // q-heads per kv-head handled by one CTA
constexpr int kRowsInFlight = 4;    // K / V rows a warp loads before using them

struct DecodeLayout {
    size_t keys, ids, flags, crow, grow, qh, sc, red, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// Dynamic shared memory of the decode kernel.
__host__ __device__ inline DecodeLayout decode_layout(int64_t nC, int wc, int wg, int G, int D)
{
    DecodeLayout L;
    const size_t nk = (size_t)(nC > 8 * (int64_t)wc ? nC : 8 * (int64_t)wc);
    const size_t maxkeys = 8 * (size_t)wg + kChunk;
    L.keys = 0;
    L.ids = align16(L.keys + 8 * nk);
    L.flags = align16(L.ids + 4 * 8 * (size_t)wc);
    L.crow = align16(L.flags + 8 * (size_t)wc);
    L.grow = align16(L.crow + 4 * (size_t)wc);
    L.qh = align16(L.grow + 4 * (size_t)wg);
    L.sc = align16(L.qh + 4 * (size_t)G * D);
    L.red = align16(L.sc + 4 * (size_t)G * maxkeys);
    L.total = align16(L.red + 4 * (size_t)kRouterWarps * G * D);
    return L;
}

// P consecutive elements widened to float32 (P = 2 or 4; 4- to 16-byte loads).
template <typename TIn, int P> struct RowLoad;
template <> struct RowLoad<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* o) {
        const uint2 r = __ldg(reinterpret_cast<const uint2*>(p));
        o[0] = __uint_as_float(r.x << 16); o[1] = __uint_as_float(r.x & 0xFFFF0000u);
        o[2] = __uint_as_float(r.y << 16); o[3] = __uint_as_float(r.y & 0xFFFF0000u);
    }
};
template <> struct RowLoad<__nv_bfloat16, 2> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* o) {
        const uint32_t r = __ldg(reinterpret_cast<const unsigned int*>(p));
        o[0] = __uint_as_float(r << 16); o[1] = __uint_as_float(r & 0xFFFF0000u);
    }
};
template <> struct RowLoad<float, 4> {
    static __device__ __forceinline__ void load(const float* p, float* o) {
        const float4 r = __ldg(reinterpret_cast<const float4*>(p));
        o[0] = r.x; o[1] = r.y; o[2] = r.z; o[3] = r.w;
    }
};
template <> struct RowLoad<float, 2> {
    static __device__ __forceinline__ void load(const float* p, float* o) {
        const float2 r = __ldg(reinterpret_cast<const float2*>(p));
        o[0] = r.x; o[1] = r.y;
    }
};

template <typename TIn> __device__ __forceinline__ float to_f32(TIn x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename TIn, int D>
__global__ void __launch_bounds__(kRouterThreads, 1)
decode_kernel(const TIn* __restrict__ q, const TIn* __restrict__ K, const TIn* __restrict__ V,
              const float* __restrict__ csum, const float* __restrict__ gsum, float* __restrict__ O,
              float* __restrict__ lse, int32_t* __restrict__ cidx, int32_t* __restrict__ gidx, int Hq, int Hkv,
              int G, int64_t T, int64_t pos, int k_c, int wc, int k_g, int wg, float scale)
{
    pdl_wait();
    pdl_trigger();
    constexpr int P = D / 32;                        // elements of a row per lane
    constexpr int R = kRowsInFlight;
    extern __shared__ __align__(16) uint8_t sm[];
    const int64_t nC = T / kChunk, nG = T / kGroup;
    const DecodeLayout L = decode_layout(nC, wc, wg, G, D);
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(sm + L.keys);
    int32_t* ids = reinterpret_cast<int32_t*>(sm + L.ids);
    uint8_t* flags = sm + L.flags;
    int32_t* crow = reinterpret_cast<int32_t*>(sm + L.crow);
    int32_t* grow = reinterpret_cast<int32_t*>(sm + L.grow);
    float* qh = reinterpret_cast<float*>(sm + L.qh);     // [G][D] the token's queries
    float* sc = reinterpret_cast<float*>(sm + L.sc);     // [G][maxkeys] scores, then weights
    float* red = reinterpret_cast<float*>(sm + L.red);   // [warps][G][D] partial outputs
    __shared__ __align__(16) float qs[D];
    __shared__ int n_valid, s_ng;
    const int maxkeys = 8 * wg + kChunk;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bg = blockIdx.x;
    const int64_t b = bg / Hkv, g = bg % Hkv;

    // The token's queries of the G heads, and their mean (the block query).
    for (int i = tid; i < G * D; i += kRouterThreads) qh[i] = to_f32<TIn>(q[(b * Hq + g * G) * D + i]);
    __syncthreads();
    for (int e = tid; e < D; e += kRouterThreads) {
        float a = 0.f;
        for (int h = 0; h < G; ++h) a += qh[h * D + e];
        qs[e] = a / (float)G;
    }
    __syncthreads();
    // Chunk and group routing of the one-token block.
    const int c0 = int(pos / kChunk);
    int32_t* gout = gidx + bg * wg;
    route_chunks_block<D>(qs, csum + bg * nC * D, c0, k_c, wc, keys, cidx + bg * wc, crow, tid);
    route_groups_block<D>(qs, gsum + bg * nG * D, crow, wc, k_g, wg, keys, ids, flags, &n_valid, grow, tid);
    __syncthreads();
    for (int i = tid; i < wg; i += kRouterThreads) gout[i] = grow[i];
    if (warp == 0) {                                 // routed groups: an ascending prefix
        int n = 0;
        for (int base = 0; base < wg; base += 32) {
            const int i = base + lane;
            n += __popc(__ballot_sync(0xFFFFFFFFu, i < wg && grow[i] >= 0));
        }
        if (lane == 0) s_ng = n;
    }
    __syncthreads();
    const int n_g = s_ng;
    const int n_keys = kGroup * n_g + int(pos - (int64_t)c0 * kChunk) + 1;
    const TIn* Kb = K + bg * T * D + lane * P;
    const TIn* Vb = V + bg * T * D + lane * P;
    // Key k: the tokens of the routed groups in order, then the own chunk's
    // tokens 64 c0 .. pos.
    auto token = [&](int k) -> int64_t {
        return k < kGroup * n_g ? (int64_t)grow[k / kGroup] * kGroup + k % kGroup
                                : (int64_t)c0 * kChunk + (k - kGroup * n_g);
    };
    // Scores: warp w takes keys w + 8 j; lane l holds elements lP .. lP+P-1
    // of the key row and of every head's query.
    float qv[kMaxG][P];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h)
#pragma unroll
        for (int e = 0; e < P; ++e) qv[h][e] = h < G ? qh[h * D + lane * P + e] : 0.f;
    for (int k0 = warp; k0 < n_keys; k0 += R * kRouterWarps) {
        float kv[R][P];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int k = k0 + r * kRouterWarps;
            if (k < n_keys) RowLoad<TIn, P>::load(Kb + token(k) * D, kv[r]);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int k = k0 + r * kRouterWarps;
            if (k >= n_keys) break;
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                if (h >= G) break;
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < P; ++e) a = fmaf(qv[h][e], kv[r][e], a);
                a = warp_sum(a);
                if (lane == 0) sc[h * maxkeys + k] = a * scale;
            }
        }
    }
    __syncthreads();
    // Softmax of each head (warp h, h + 8, ...): weights in place, lse.
    for (int h = warp; h < G; h += kRouterWarps) {
        float* s = sc + h * maxkeys;
        float m = -INFINITY;
        for (int k = lane; k < n_keys; k += 32) m = fmaxf(m, s[k]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        float l = 0.f;
        for (int k = lane; k < n_keys; k += 32) {
            const float w = expf(s[k] - m);
            s[k] = w;
            l += w;
        }
        l = warp_sum(l);
        const float inv = 1.0f / l;
        for (int k = lane; k < n_keys; k += 32) s[k] *= inv;
        if (lane == 0) lse[b * Hq + g * G + h] = m + logf(l);
    }
    __syncthreads();
    // O = P V: warp w accumulates keys w + 8 j for every head, then the 8
    // warps' partial sums are added.
    float acc[kMaxG][P];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h)
#pragma unroll
        for (int e = 0; e < P; ++e) acc[h][e] = 0.f;
    for (int k0 = warp; k0 < n_keys; k0 += R * kRouterWarps) {
        float vv[R][P];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int k = k0 + r * kRouterWarps;
            if (k < n_keys) RowLoad<TIn, P>::load(Vb + token(k) * D, vv[r]);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int k = k0 + r * kRouterWarps;
            if (k >= n_keys) break;
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                if (h >= G) break;
                const float w = sc[h * maxkeys + k];
#pragma unroll
                for (int e = 0; e < P; ++e) acc[h][e] = fmaf(w, vv[r][e], acc[h][e]);
            }
        }
    }
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
        if (h >= G) break;
#pragma unroll
        for (int e = 0; e < P; ++e) red[(warp * G + h) * D + lane * P + e] = acc[h][e];
    }
    __syncthreads();
    for (int i = tid; i < G * D; i += kRouterThreads) {
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < kRouterWarps; ++w) a += red[w * G * D + i];
        O[(b * Hq + g * G) * D + i] = a;
    }
}

template <typename TIn, int D>
cudaError_t launch(const Shape& s, int64_t pos, const void* q, const void* K, const void* V, const float* csum,
                   const float* gsum, float* O, float* lse, int32_t* cidx, int32_t* gidx, cudaStream_t st)
{
    const size_t smem = decode_layout(s.nC, s.wc, s.wg, s.G, D).total;
    auto k = decode_kernel<TIn, D>;
    cudaError_t e = allow_smem(k, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3((unsigned)(s.B * s.Hkv)), dim3(kRouterThreads), smem, st,
                      static_cast<const TIn*>(q), static_cast<const TIn*>(K), static_cast<const TIn*>(V), csum,
                      gsum, O, lse, cidx, gidx, s.Hq, s.Hkv, s.G, s.T, pos, s.k_c, s.wc, s.k_g, s.wg, s.scale);
}

}  // namespace

size_t decode_smem(const Shape& s) { return decode_layout(s.nC, s.wc, s.wg, s.G, s.d).total; }
int decode_max_heads() { return kMaxG; }

cudaError_t launch_decode(const Shape& s, int64_t pos, const void* q, const void* K, const void* V,
                          const float* csum, const float* gsum, float* O, float* lse, int32_t* cidx,
                          int32_t* gidx, cudaStream_t st)
{
    if (s.dtype == HGA_BF16)
        return s.d == 128 ? launch<__nv_bfloat16, 128>(s, pos, q, K, V, csum, gsum, O, lse, cidx, gidx, st)
                          : launch<__nv_bfloat16, 64>(s, pos, q, K, V, csum, gsum, O, lse, cidx, gidx, st);
    return s.d == 128 ? launch<float, 128>(s, pos, q, K, V, csum, gsum, O, lse, cidx, gidx, st)
                      : launch<float, 64>(s, pos, q, K, V, csum, gsum, O, lse, cidx, gidx, st);
}

}  // namespace hga
