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
// One thread-block cluster of kS = 8 CTAs per (batch, kv-head), 256 threads
// each.  A decode step is a chain of dependent memory round trips (query ->
// chunk scores -> group scores -> K / V rows), so the cluster splits every
// link of the chain:
//   * chunk and group scoring: CTA r scores the r-th eighth of the
//     candidates and writes the keys into every peer's shared memory
//     (distributed shared memory); after a cluster barrier each CTA holds
//     all keys and runs the same selection, so all hold the same routing;
//   * attention: the keys come in 8-token units (the own chunk's tokens up
//     to pos, then the routed groups, 8 contiguous rows each); CTA r takes
//     units r, r + 8, ..., stages them into shared memory with bulk copies
//     (tiles of 8 units, one mbarrier) and keeps a running softmax per head;
//     the own chunk's unit is fetched at kernel start, before the routing;
//   * combine: every CTA writes (max, sum, unnormalised O) of each head into
//     CTA 0's shared memory; CTA 0 merges them (log-sum-exp) and stores O
//     and lse.
// Float32 arithmetic throughout.
#include "hga_internal.cuh"
#include "router_core.cuh"
#include "sm100.cuh"

namespace hga {
namespace {

using namespace rt;
using namespace sm100;

constexpr int kS = 8;                       // CTAs per (batch, kv-head): one cluster
constexpr int kMaxG = 8;                    // q-heads per kv-head
constexpr int kTileUnits = 8;               // 8-token units a CTA stages at once
constexpr int kTileRows = kTileUnits * kGroup;
constexpr int kSiteOwn = 0x301, kSiteTile = 0x302;   // bounded-wait sites

struct DecodeLayout {
    size_t ckeys, gkeys, ids, flags, crow, grow, qh, kv, sc, hs, part, pvred, bar, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }
__host__ __device__ inline size_t align128(size_t x) { return (x + 127) & ~size_t(127); }

// Floats per CTA in the combine area: O [G][D], then max [G] and sum [G]
// padded to a multiple of 4 (each CTA's block starts 16-byte aligned).
__host__ __device__ inline int part_stride(int G, int D) { return G * D + ((2 * G + 3) & ~3); }

// Dynamic shared memory of the decode kernel (el = bytes per K / V element).
//   ckeys [nC] / gkeys [8 wc]   selection keys of chunks / groups (u64)
//   ids [8 wc], flags [8 wc]    group candidates, their keep flags
//   crow [wc], grow [wg]        the routing rows
//   qh [G][D]                   the token's queries (float)
//   kv                          K tile [64][D] then V tile [64][D] (input dtype)
//   sc [G][64]                  scores, then weights, of the tile
//   hs [3][G]                   running max, sum and rescale factor per head
//   part [kS][part_stride]      per-CTA O [G][D], max [G], sum [G] read by CTA 0
//   pvred [256] float4          P V partial sums of the row slices
//   bar                         two mbarriers (own unit, tiles)
__host__ __device__ inline DecodeLayout decode_layout(int64_t nC, int wc, int wg, int G, int D, int el)
{
    DecodeLayout L;
    L.ckeys = 0;
    L.gkeys = align16(L.ckeys + 8 * (size_t)(nC > 0 ? nC : 1));
    L.ids = align16(L.gkeys + 8 * 8 * (size_t)wc);
    L.flags = align16(L.ids + 4 * 8 * (size_t)wc);
    L.crow = align16(L.flags + 8 * (size_t)wc);
    L.grow = align16(L.crow + 4 * (size_t)wc);
    L.qh = align16(L.grow + 4 * (size_t)wg);
    L.kv = align128(L.qh + 4 * (size_t)G * D);
    L.sc = align16(L.kv + 2 * (size_t)kTileRows * D * el);
    L.hs = align16(L.sc + 4 * (size_t)G * kTileRows);
    L.part = align16(L.hs + 4 * 3 * (size_t)G);
    L.pvred = align16(L.part + 4 * (size_t)kS * part_stride(G, D));
    L.bar = align16(L.pvred + 16 * (size_t)kRouterThreads);
    L.total = align16(L.bar + 16);
    return L;
}

// P consecutive elements of a shared-memory row widened to float32.
template <typename TIn, int P> __device__ __forceinline__ void smem_row(const TIn* p, float* o);
template <> __device__ __forceinline__ void smem_row<__nv_bfloat16, 4>(const __nv_bfloat16* p, float* o)
{
    const uint2 r = *reinterpret_cast<const uint2*>(p);
    o[0] = __uint_as_float(r.x << 16); o[1] = __uint_as_float(r.x & 0xFFFF0000u);
    o[2] = __uint_as_float(r.y << 16); o[3] = __uint_as_float(r.y & 0xFFFF0000u);
}
template <> __device__ __forceinline__ void smem_row<__nv_bfloat16, 2>(const __nv_bfloat16* p, float* o)
{
    const uint32_t r = *reinterpret_cast<const uint32_t*>(p);
    o[0] = __uint_as_float(r << 16); o[1] = __uint_as_float(r & 0xFFFF0000u);
}
template <> __device__ __forceinline__ void smem_row<float, 4>(const float* p, float* o)
{
    const float4 r = *reinterpret_cast<const float4*>(p);
    o[0] = r.x; o[1] = r.y; o[2] = r.z; o[3] = r.w;
}
template <> __device__ __forceinline__ void smem_row<float, 2>(const float* p, float* o)
{
    const float2 r = *reinterpret_cast<const float2*>(p);
    o[0] = r.x; o[1] = r.y;
}

template <typename TIn> __device__ __forceinline__ float to_f32(TIn x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// keys[b, e) of this CTA, written into the same slots of every peer.
__device__ __forceinline__ void push_keys(unsigned long long* keys, int b, int e, uint32_t rank, int tid)
{
    for (int i = b + tid; i < e; i += kRouterThreads) {
        const unsigned long long v = keys[i];
        const uint32_t a = smem_u32(keys + i);
#pragma unroll
        for (uint32_t p = 0; p < kS; ++p)
            if (p != rank) st_cluster_u64(peer_addr(a, p), v);
    }
}

template <typename TIn, int D>
__global__ void __launch_bounds__(kRouterThreads, 2)
decode_kernel(const TIn* __restrict__ q, const TIn* __restrict__ K, const TIn* __restrict__ V,
              const float* __restrict__ csum, const float* __restrict__ gsum, float* __restrict__ O,
              float* __restrict__ lse, int32_t* __restrict__ cidx, int32_t* __restrict__ gidx, int Hq, int Hkv,
              int G, int64_t T, int64_t cap, int64_t pos, int k_c, int wc, int k_g, int wg, float scale)
{
    constexpr int P = D / 32;                        // elements of a row per lane
    constexpr uint32_t kRowBytes = D * sizeof(TIn);
    extern __shared__ __align__(128) uint8_t sm[];
    const int64_t nC = T / kChunk, nCs = cap / kChunk, nGs = cap / kGroup;
    const DecodeLayout L = decode_layout(nC, wc, wg, G, D, (int)sizeof(TIn));
    unsigned long long* ckeys = reinterpret_cast<unsigned long long*>(sm + L.ckeys);
    unsigned long long* gkeys = reinterpret_cast<unsigned long long*>(sm + L.gkeys);
    int32_t* ids = reinterpret_cast<int32_t*>(sm + L.ids);
    uint8_t* flags = sm + L.flags;
    int32_t* crow = reinterpret_cast<int32_t*>(sm + L.crow);
    int32_t* grow = reinterpret_cast<int32_t*>(sm + L.grow);
    float* qh = reinterpret_cast<float*>(sm + L.qh);
    TIn* kt = reinterpret_cast<TIn*>(sm + L.kv);
    TIn* vt = kt + kTileRows * D;
    float* sc = reinterpret_cast<float*>(sm + L.sc);
    float* hm = reinterpret_cast<float*>(sm + L.hs);   // running max per head
    float* hl = hm + G;                                // running sum
    float* ha = hl + G;                                // rescale of the current tile
    float* part = reinterpret_cast<float*>(sm + L.part);
    const uint32_t bar_own = smem_u32(sm + L.bar), bar_tile = bar_own + 8;
    __shared__ __align__(16) float qs[D];
    __shared__ int s_cnt, s_ng;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t r = cluster_rank();
    const int64_t bg = blockIdx.x / kS;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    const TIn* Kb = K + bg * cap * D;                // K / V rows of (b, g): cap apart
    const TIn* Vb = V + bg * cap * D;

    if (tid == 0) {
        mbar_init(bar_own, 1);
        mbar_init(bar_tile, 1);
        fence_mbar_init();
    }
    if (tid < G) {
        hm[tid] = -INFINITY;
        hl[tid] = 0.f;
    }
    pdl_wait();
    pdl_trigger();

    // The own chunk's tokens 64 c0 .. pos form units 0 .. n_ou-1 (n_ou <= 8):
    // CTA r's is unit r, slot 0 of its first tile; fetch it now.  Also bring
    // this CTA's slice of the chunk summaries into L2 ahead of the scoring.
    const int c0 = int(pos / kChunk);
    const int own_rows = int(pos - (int64_t)c0 * kChunk) + 1;
    const int n_ou = (own_rows + kGroup - 1) / kGroup;
    const bool has_own = (int)r < n_ou;
    const int own_r = has_own ? min(kGroup, own_rows - kGroup * (int)r) : 0;
    const bool score_c = k_c > 0 && k_c < c0;
    const int cb = (int)r * c0 / kS, ce = ((int)r + 1) * c0 / kS;
    const float* cs = csum + bg * nCs * D;
    if (tid == 0) {
        if (has_own) {
            const int64_t t0 = (int64_t)c0 * kChunk + kGroup * r;
            mbar_expect_tx(bar_own, 2 * own_r * kRowBytes);
            bulk_load(smem_u32(kt), Kb + t0 * D, own_r * kRowBytes, bar_own);
            bulk_load(smem_u32(vt), Vb + t0 * D, own_r * kRowBytes, bar_own);
        }
        if (score_c && ce > cb) bulk_prefetch_l2(cs + (int64_t)cb * D, (uint32_t)(ce - cb) * D * 4u);
    }
    // The token's queries of the G heads (loads overlap the cluster barrier).
    for (int i = tid; i < G * D; i += kRouterThreads) qh[i] = to_f32<TIn>(q[(b * Hq + g * G) * D + i]);
    cluster_sync();                                  // all CTAs run; barriers initialised; qh complete

    // The block query: mean of the G heads' queries.
    for (int e = tid; e < D; e += kRouterThreads) {
        float a = 0.f;
        for (int h = 0; h < G; ++h) a += qh[h * D + e];
        qs[e] = a / (float)G;
    }
    __syncthreads();

    // a3: chunk routing.  CTA r scores chunks [r c0 / 8, (r+1) c0 / 8).
    if (score_c) {
        score_candidates<D>(qs, ce - cb, [&](int c, const float*& row) { row = cs + (int64_t)(cb + c) * D; return cb + c; },
                            ckeys + cb, warp, lane);
        __syncthreads();
        push_keys(ckeys, cb, ce, r, tid);
    }
    cluster_sync();
    if (score_c) {
        select_chunks(ckeys, c0, k_c, wc, crow, r == 0 ? cidx + bg * wc : nullptr, warp, lane);
    } else {
        for (int i = tid; i < wc; i += kRouterThreads) {
            const int32_t v = i < c0 ? i : -1;
            crow[i] = v;
            if (r == 0) cidx[bg * wc + i] = v;
        }
    }
    __syncthreads();

    // a4: group routing over the 8 groups of every routed chunk.  CTA r
    // scores candidates [r n / 8, (r+1) n / 8).
    if (warp == 0) {
        const int n = prefix_count(crow, wc, lane);
        if (lane == 0) s_cnt = n;
    }
    __syncthreads();
    const int n_cand = s_cnt * kGroupsPerChunk;
    for (int i = tid; i < n_cand; i += kRouterThreads)
        ids[i] = crow[i / kGroupsPerChunk] * kGroupsPerChunk + i % kGroupsPerChunk;
    __syncthreads();
    const bool score_g = k_g > 0 && k_g < n_cand;
    if (score_g) {
        const int gb = (int)r * n_cand / kS, ge = ((int)r + 1) * n_cand / kS;
        const float* gs = gsum + bg * nGs * D;
        score_candidates<D>(qs, ge - gb,
                            [&](int c, const float*& row) { row = gs + (int64_t)ids[gb + c] * D; return ids[gb + c]; },
                            gkeys + gb, warp, lane);
        __syncthreads();
        push_keys(gkeys, gb, ge, r, tid);
    }
    cluster_sync();
    if (score_g) {
        select_groups(gkeys, ids, n_cand, k_g, flags, grow, wg, tid);
    } else {
        for (int i = tid; i < wg; i += kRouterThreads) grow[i] = i < n_cand ? ids[i] : -1;
    }
    __syncthreads();
    if (r == 0)
        for (int i = tid; i < wg; i += kRouterThreads) gidx[bg * wg + i] = grow[i];
    if (warp == 0) {
        const int n = prefix_count(grow, wg, lane);
        if (lane == 0) s_ng = n;
    }
    __syncthreads();

    // Attention.  Units: 0 .. n_ou-1 the own chunk's, then the routed groups;
    // CTA r takes units r + 8 j, tile t holding j = 8 t .. 8 t + 7 (slot j - 8 t).
    const int n_u = n_ou + s_ng;
    const int my_units = n_u > (int)r ? (n_u - (int)r + kS - 1) / kS : 0;
    const int n_tiles = (my_units + kTileUnits - 1) / kTileUnits;
    // Rows of a partial own unit past pos are zero in the V tile (their
    // weight is 0, and 0 times stale shared memory could be NaN).
    if (has_own && own_r < kGroup) {
        for (int i = own_r * D + tid; i < kGroup * D; i += kRouterThreads) vt[i] = TIn(0.f);
        fence_async_smem();                          // ordered before later bulk copies into the slot
    }
    float qv[kMaxG][P];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h)
#pragma unroll
        for (int e = 0; e < P; ++e) qv[h][e] = h < G ? qh[h * D + lane * P + e] : 0.f;
    // P V: the outputs [G][D] in nq quads of 4; thread tid takes quad
    // tid % nq for the rows j = tid / nq (mod nh) of every tile, nh row
    // slices in all; the slices' sums are added after the last tile.
    const int nq = G * D / 4;
    const int nh = kRouterThreads / nq;
    const int slice = tid / nq;
    const bool pv_on = slice < nh;
    const int i4 = 4 * (tid % nq);
    const int ph = i4 / D, pe = i4 % D;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
        const int slots = min(kTileUnits, my_units - t * kTileUnits);
        if (tid == 0) {
            uint32_t bytes = 0;
            for (int i = 0; i < slots; ++i)
                if ((int)r + kS * (t * kTileUnits + i) >= n_ou) bytes += kGroup * kRowBytes;
            mbar_expect_tx(bar_tile, 2 * bytes);
            for (int i = 0; i < slots; ++i) {
                const int u = (int)r + kS * (t * kTileUnits + i);
                if (u < n_ou) continue;
                const int64_t t0 = (int64_t)grow[u - n_ou] * kGroup;
                bulk_load(smem_u32(kt + i * kGroup * D), Kb + t0 * D, kGroup * kRowBytes, bar_tile);
                bulk_load(smem_u32(vt + i * kGroup * D), Vb + t0 * D, kGroup * kRowBytes, bar_tile);
            }
        }
        bool w = true;
        if (t == 0 && has_own) w = mbar_wait(bar_own, 0, kSiteOwn);
        w = mbar_wait(bar_tile, t & 1, kSiteTile) && w;
        if (!__syncthreads_and(w)) {                 // a copy did not land in time
            ok = false;
            break;
        }
        // Scores of the tile's rows: warp w takes rows w, w + 8, ...
        const int nrows = slots * kGroup;
        for (int j = warp; j < nrows; j += kRouterWarps) {
            const bool valid = !(t == 0 && j < kGroup && has_own) || j < own_r;
            float kv[P];
            smem_row<TIn, P>(kt + j * D + lane * P, kv);
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                if (h >= G) break;
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < P; ++e) a = fmaf(qv[h][e], kv[e], a);
                a = warp_sum(a);
                if (lane == 0) sc[h * kTileRows + j] = valid ? a * scale : -INFINITY;
            }
        }
        __syncthreads();
        // Running softmax per head (warp h): weights of the tile, rescale.
        for (int h = warp; h < G; h += kRouterWarps) {
            float* s = sc + h * kTileRows;
            float mt = -INFINITY;
            for (int j = lane; j < nrows; j += 32) mt = fmaxf(mt, s[j]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, o));
            const float mo = hm[h], mn = fmaxf(mo, mt);
            float ls = 0.f;
            for (int j = lane; j < nrows; j += 32) {
                const float p = expf(s[j] - mn);
                s[j] = p;
                ls += p;
            }
            ls = warp_sum(ls);
            if (lane == 0) {
                const float a = expf(mo - mn);
                ha[h] = a;
                hl[h] = hl[h] * a + ls;
                hm[h] = mn;
            }
        }
        __syncthreads();
        if (pv_on) {
            const float a = ha[ph];
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] *= a;
            const float* wts = sc + ph * kTileRows;
            for (int j = slice; j < nrows; j += nh) {
                float v[4];
                smem_row<TIn, 4>(vt + j * D + pe, v);
                const float p = wts[j];
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[k] = fmaf(p, v[k], acc[k]);
            }
        }
        __syncthreads();                             // the tile is free for the next copies
    }

    // The row slices' partial sums, added in slice order by slice 0.
    float4* pvred = reinterpret_cast<float4*>(sm + L.pvred);
    if (pv_on && slice > 0) pvred[(slice - 1) * nq + tid % nq] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    const bool pv0 = slice == 0;
    if (pv0) {
        for (int sl = 1; sl < nh; ++sl) {
            const float4 v = pvred[(sl - 1) * nq + tid];
            acc[0] += v.x;
            acc[1] += v.y;
            acc[2] += v.z;
            acc[3] += v.w;
        }
    }

    // Combine in CTA 0: O = sum_r O_r e^(m_r - M) / sum_r l_r e^(m_r - M).
    const int stride = part_stride(G, D);
    float* mine = part + (int)r * stride;
    if (tid < G) {
        st_cluster_f32(peer_addr(smem_u32(mine + G * D + tid), 0), ok ? hm[tid] : -INFINITY);
        st_cluster_f32(peer_addr(smem_u32(mine + G * D + G + tid), 0), ok ? hl[tid] : 0.f);
    }
    if (pv0) {
        const float z = ok ? 1.f : 0.f;
        st_cluster_v4(peer_addr(smem_u32(mine + i4), 0), acc[0] * z, acc[1] * z, acc[2] * z, acc[3] * z);
    }
    cluster_sync();
    if (r == 0 && pv0) {
        float M = -INFINITY;
#pragma unroll
        for (int c = 0; c < kS; ++c) M = fmaxf(M, part[c * stride + G * D + ph]);
        float Ls = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < kS; ++c) {
            const float* pc = part + c * stride;
            const float f = expf(pc[G * D + ph] - M);
            Ls = fmaf(pc[G * D + G + ph], f, Ls);
            const float4 oc = *reinterpret_cast<const float4*>(pc + i4);
            o[0] = fmaf(oc.x, f, o[0]);
            o[1] = fmaf(oc.y, f, o[1]);
            o[2] = fmaf(oc.z, f, o[2]);
            o[3] = fmaf(oc.w, f, o[3]);
        }
        const float inv = 1.0f / Ls;
        *reinterpret_cast<float4*>(O + (b * Hq + g * G) * D + i4) =
            make_float4(o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
        if (pe == 0) lse[b * Hq + g * G + ph] = M + logf(Ls);
    }
}

template <typename TIn, int D>
cudaError_t launch(const Shape& s, int64_t pos, const void* q, const void* K, const void* V, const float* csum,
                   const float* gsum, float* O, float* lse, int32_t* cidx, int32_t* gidx, cudaStream_t st)
{
    const size_t smem = decode_layout(s.nC, s.wc, s.wg, s.G, D, (int)sizeof(TIn)).total;
    auto k = decode_kernel<TIn, D>;
    cudaError_t e = allow_smem(k, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(s.B * s.Hkv * kS));
    cfg.blockDim = dim3(kRouterThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    // An 8-CTA cluster per (batch, kv-head); programmatic dependent launch,
    // so that a step's launch overlaps the previous kernel's tail (the
    // kernel reads no global memory before its griddepcontrol.wait).
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k, static_cast<const TIn*>(q), static_cast<const TIn*>(K),
                              static_cast<const TIn*>(V), csum, gsum, O, lse, cidx, gidx, s.Hq, s.Hkv, s.G, s.T,
                              s.cap, pos, s.k_c, s.wc, s.k_g, s.wg, s.scale);
}

}  // namespace

size_t decode_smem(const Shape& s)
{
    return decode_layout(s.nC, s.wc, s.wg, s.G, s.d, s.dtype == HGA_BF16 ? 2 : 4).total;
}
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

// Status word of the decode kernel's bounded waits (0 = none ran out).
int decode_status(bool clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, sm100::g_status, sizeof v) != cudaSuccess) return -1;
    if (clear && v) {
        const int z = 0;
        cudaMemcpyToSymbol(sm100::g_status, &z, sizeof z);
    }
    return v;
}

}  // namespace hga
