// attn_simt.cu -- a5 / a6 routed attention on the CUDA cores (float32 FMA).
//
// Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com),
// section "What HGA does differently": the attention loads only the exact
// token K/V of the selected groups; gradients reach Q/K/V as in the dense
// case because the router has no learned weights; older KV is detached, so
// the backward keeps key gradients for segment tokens only.
//
// This is the float32 path (inputs of dtype HGA_FP32 must match the oracle
// to 1e-4, which rules out reduced-precision tensor-core products), written
// for any input type.  One CTA owns one (batch, q-head, query block): 64
// query rows.  Keys are visited in tiles of 64: ceil(n_groups / 8) tiles of
// routed groups (8 groups each), then the own chunk with the token-causal
// mask.  Thread (ty, tx) of a 16 x 16 grid owns rows 4ty..4ty+3 and the
// columns tx + 16c, which keeps the shared-memory reads conflict-free.
#include "check.cuh"
#include "hga_internal.cuh"

namespace hga {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D> __host__ __device__ constexpr int padded() { return D + 1; }

// Copy 64 rows of a [.][D] tensor into shared memory [64][D+1] as float32.
// row_src(r) gives the global row (or nullptr for a zero row).
template <typename TIn, int D, typename RowFn>
__device__ __forceinline__ void load_tile(float* dst, RowFn row_src)
{
    constexpr int E = Vec16<TIn>::E, V16 = D / E, DP = padded<D>();
    for (int i = threadIdx.x; i < kTile * V16; i += kThreads) {
        const int r = i / V16, v = i % V16;
        const TIn* src = row_src(r);
        float x[E];
        if (src) Vec16<TIn>::load(src + v * E, x);
        else {
#pragma unroll
            for (int e = 0; e < E; ++e) x[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < E; ++e) dst[r * DP + v * E + e] = x[e];
    }
}

// s[a][c] = sum_e A[4ty+a][e] * B[tx+16c][e]
template <int D>
__device__ __forceinline__ void tile_dot(const float* A, const float* Bm, int ty, int tx, float s[4][4])
{
    constexpr int DP = padded<D>();
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) s[a][c] = 0.f;
#pragma unroll 4
    for (int e = 0; e < D; ++e) {
        float x[4], y[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) x[a] = A[(4 * ty + a) * DP + e];
#pragma unroll
        for (int c = 0; c < 4; ++c) y[c] = Bm[(tx + 16 * c) * DP + e];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) s[a][c] = fmaf(x[a], y[c], s[a][c]);
    }
}

__device__ __forceinline__ float half_warp_max(float v)
{
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}
__device__ __forceinline__ float half_warp_sum(float v)
{
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Number of valid (non -1) entries of an index row; they form a prefix.
// In checked builds the n entries used are range-checked (0 <= j < limit,
// limit = 8 * own chunk), which also catches a -1 inside the prefix.
__device__ __forceinline__ int count_valid(const int32_t* row, int w, int* s_groups, int64_t limit, int site)
{
    __shared__ int n;
    if (threadIdx.x == 0) n = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < w; i += kThreads) {
        const int32_t j = row[i];
        s_groups[i] = j;
        if (j >= 0) atomicAdd(&n, 1);
    }
    __syncthreads();
    if (chk::kEnabled) {
        for (int i = threadIdx.x; i < n; i += kThreads) s_groups[i] = chk::group(s_groups[i], limit, site);
        __syncthreads();
    }
    return n;
}

// Global token of key row kr (0..63) of key tile `tile`, or -1 if masked out
// for every query (padding of a partial routed tile).
__device__ __forceinline__ int64_t key_token(int tile, int n_routed_tiles, int n_groups,
                                             const int* s_groups, int64_t own_start, int kr)
{
    if (tile < n_routed_tiles) {
        const int gi = tile * 8 + kr / kGroup;
        return gi < n_groups ? (int64_t)s_groups[gi] * kGroup + kr % kGroup : -1;
    }
    return own_start + kr;
}

// ---------------------------------------------------------------- forward --
template <typename TIn, int D>
__global__ void __launch_bounds__(kThreads)
attn_fwd_simt_kernel(const TIn* __restrict__ Q, const TIn* __restrict__ K,
                     const TIn* __restrict__ V, const int32_t* __restrict__ gidx,
                     float* __restrict__ O, float* __restrict__ lse,
                     int Hq, int Hkv, int G, int64_t T_hist, int64_t T_seg, int64_t nQB, int64_t cap, int wg,
                     float scale_log2)
{
    constexpr int DP = padded<D>(), NC = D / 16;
    extern __shared__ float sm[];
    float* Qs = sm;
    float* Ks = Qs + kTile * DP;
    float* Vs = Ks + kTile * DP;
    float* Ps = Vs + kTile * DP;                  // [64][65]
    int* s_groups = reinterpret_cast<int*>(Ps + kTile * (kTile + 1));

    const int64_t bhq = blockIdx.x;               // ((b*Hq)+h)*nQB + qb
    const int64_t qb = bhq % nQB, bh = bhq / nQB;
    const int64_t b = bh / Hq, h = bh % Hq, g = h / G;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;

    const TIn* Qrow0 = Q + (bh * T_seg + qb * kTile) * D;
    const TIn* Kh = K + (b * Hkv + g) * cap * D;     // K / V rows of (b, g): cap apart
    const TIn* Vh = V + (b * Hkv + g) * cap * D;
    const int n_groups = count_valid(gidx + ((b * Hkv + g) * nQB + qb) * wg, wg, s_groups,
                                     (T_hist + qb * kTile) / kGroup, chk::kSiteSimtFwd);
    const int n_routed_tiles = (n_groups + 7) / 8;
    const int64_t own_start = T_hist + qb * kTile;

    load_tile<TIn, D>(Qs, [&](int r) { return Qrow0 + (int64_t)r * D; });

    float m[4], l[4], acc[4][NC];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        m[a] = -INFINITY;
        l[a] = 0.f;
#pragma unroll
        for (int j = 0; j < NC; ++j) acc[a][j] = 0.f;
    }

    for (int tile = 0; tile <= n_routed_tiles; ++tile) {
        const bool own = tile == n_routed_tiles;
        __syncthreads();
        load_tile<TIn, D>(Ks, [&](int r) {
            const int64_t t = key_token(tile, n_routed_tiles, n_groups, s_groups, own_start, r);
            return t >= 0 ? Kh + t * D : nullptr;
        });
        load_tile<TIn, D>(Vs, [&](int r) {
            const int64_t t = key_token(tile, n_routed_tiles, n_groups, s_groups, own_start, r);
            return t >= 0 ? Vh + t * D : nullptr;
        });
        __syncthreads();
        float s[4][4];
        tile_dot<D>(Qs, Ks, ty, tx, s);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int row = 4 * ty + a;
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int col = tx + 16 * c;
                const bool ok = own ? (col <= row) : (tile * 8 + col / kGroup < n_groups);
                s[a][c] = ok ? s[a][c] * scale_log2 : -INFINITY;
                mx = fmaxf(mx, s[a][c]);
            }
            mx = half_warp_max(mx);
            const float m_new = fmaxf(m[a], mx);
            const float alpha = exp2f(m[a] - m_new);
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float pv = exp2f(s[a][c] - m_new);
                rs += pv;
                Ps[row * (kTile + 1) + tx + 16 * c] = pv;
            }
            rs = half_warp_sum(rs);
            l[a] = l[a] * alpha + rs;
            m[a] = m_new;
#pragma unroll
            for (int j = 0; j < NC; ++j) acc[a][j] *= alpha;
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < kTile; ++kk) {
            float pv[4], vv[NC];
#pragma unroll
            for (int a = 0; a < 4; ++a) pv[a] = Ps[(4 * ty + a) * (kTile + 1) + kk];
#pragma unroll
            for (int j = 0; j < NC; ++j) vv[j] = Vs[kk * DP + tx + 16 * j];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int j = 0; j < NC; ++j) acc[a][j] = fmaf(pv[a], vv[j], acc[a][j]);
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int64_t row = bh * T_seg + qb * kTile + 4 * ty + a;
        const float inv = 1.f / l[a];
#pragma unroll
        for (int j = 0; j < NC; ++j) O[row * D + tx + 16 * j] = acc[a][j] * inv;
        if (tx == 0) lse[row] = (m[a] + log2f(l[a])) * kLn2;
    }
}

// --------------------------------------------------------------- backward --
// D_row = sum_e dO[row][e] * O[row][e], one warp per row.
template <typename TIn, int D>
__global__ void __launch_bounds__(256)
bwd_rowdot_kernel(const float* __restrict__ O, const TIn* __restrict__ dO, float* __restrict__ Drow,
                  int64_t rows)
{
    const int64_t row = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float a = 0.f;
    for (int e = lane; e < D; e += 32) a += O[row * D + e] * static_cast<float>(dO[row * D + e]);
    a = warp_sum(a);
    if (lane == 0) Drow[row] = a;
}

template <typename TIn, int D>
__global__ void __launch_bounds__(kThreads)
attn_bwd_simt_kernel(const TIn* __restrict__ Q, const TIn* __restrict__ K,
                     const TIn* __restrict__ V, const float* __restrict__ lse,
                     const TIn* __restrict__ dO, const float* __restrict__ Drow,
                     const int32_t* __restrict__ gidx, float* __restrict__ dQ,
                     float* __restrict__ dK_seg, float* __restrict__ dV_seg,
                     int Hq, int Hkv, int G, int64_t T_hist, int64_t T_seg, int64_t nQB, int64_t cap, int wg,
                     float scale, float scale_log2)
{
    constexpr int DP = padded<D>(), NC = D / 16, PP = kTile + 1;
    extern __shared__ float sm[];
    float* Qs = sm;
    float* dOs = Qs + kTile * DP;
    float* Ks = dOs + kTile * DP;
    float* Vs = Ks + kTile * DP;
    float* Ps = Vs + kTile * DP;                  // [64][65]
    float* dSs = Ps + kTile * PP;                 // [64][65]
    int* s_groups = reinterpret_cast<int*>(dSs + kTile * PP);

    const int64_t bhq = blockIdx.x;
    const int64_t qb = bhq % nQB, bh = bhq / nQB;
    const int64_t b = bh / Hq, h = bh % Hq, g = h / G;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;

    const int64_t row0 = bh * T_seg + qb * kTile;
    const TIn* Kh = K + (b * Hkv + g) * cap * D;     // K / V rows of (b, g): cap apart
    const TIn* Vh = V + (b * Hkv + g) * cap * D;
    float* dKh = dK_seg + (b * Hkv + g) * T_seg * D;
    float* dVh = dV_seg + (b * Hkv + g) * T_seg * D;
    const int n_groups = count_valid(gidx + ((b * Hkv + g) * nQB + qb) * wg, wg, s_groups,
                                     (T_hist + qb * kTile) / kGroup, chk::kSiteSimtBwd);
    const int n_routed_tiles = (n_groups + 7) / 8;
    const int64_t own_start = T_hist + qb * kTile;

    load_tile<TIn, D>(Qs, [&](int r) { return Q + (row0 + r) * D; });
    load_tile<TIn, D>(dOs, [&](int r) { return dO + (row0 + r) * D; });
    float lse2[4], Dr[4], dq[4][NC];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        lse2[a] = lse[row0 + 4 * ty + a] * kLog2e;
        Dr[a] = Drow[row0 + 4 * ty + a];
#pragma unroll
        for (int j = 0; j < NC; ++j) dq[a][j] = 0.f;
    }

    for (int tile = 0; tile <= n_routed_tiles; ++tile) {
        const bool own = tile == n_routed_tiles;
        __syncthreads();
        load_tile<TIn, D>(Ks, [&](int r) {
            const int64_t t = key_token(tile, n_routed_tiles, n_groups, s_groups, own_start, r);
            return t >= 0 ? Kh + t * D : nullptr;
        });
        load_tile<TIn, D>(Vs, [&](int r) {
            const int64_t t = key_token(tile, n_routed_tiles, n_groups, s_groups, own_start, r);
            return t >= 0 ? Vh + t * D : nullptr;
        });
        __syncthreads();
        float s[4][4], dp[4][4];
        tile_dot<D>(Qs, Ks, ty, tx, s);
        tile_dot<D>(dOs, Vs, ty, tx, dp);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int row = 4 * ty + a;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int col = tx + 16 * c;
                const bool ok = own ? (col <= row) : (tile * 8 + col / kGroup < n_groups);
                const float p = ok ? exp2f(s[a][c] * scale_log2 - lse2[a]) : 0.f;
                Ps[row * PP + col] = p;
                dSs[row * PP + col] = p * (dp[a][c] - Dr[a]);
            }
        }
        __syncthreads();
        // dQ += dS K
#pragma unroll 4
        for (int kk = 0; kk < kTile; ++kk) {
            float ds[4], kv[NC];
#pragma unroll
            for (int a = 0; a < 4; ++a) ds[a] = dSs[(4 * ty + a) * PP + kk];
#pragma unroll
            for (int j = 0; j < NC; ++j) kv[j] = Ks[kk * DP + tx + 16 * j];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int j = 0; j < NC; ++j) dq[a][j] = fmaf(ds[a], kv[j], dq[a][j]);
        }
        // dV = P^T dO and dK = dS^T Q for this thread's 4 key rows.
        float dv[4][NC], dk[4][NC];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int j = 0; j < NC; ++j) dv[a][j] = dk[a][j] = 0.f;
#pragma unroll 2
        for (int i = 0; i < kTile; ++i) {
            float pv[4], dsv[4], go[NC], qv[NC];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                pv[a] = Ps[i * PP + 4 * ty + a];
                dsv[a] = dSs[i * PP + 4 * ty + a];
            }
#pragma unroll
            for (int j = 0; j < NC; ++j) {
                go[j] = dOs[i * DP + tx + 16 * j];
                qv[j] = Qs[i * DP + tx + 16 * j];
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int j = 0; j < NC; ++j) {
                    dv[a][j] = fmaf(pv[a], go[j], dv[a][j]);
                    dk[a][j] = fmaf(dsv[a], qv[j], dk[a][j]);
                }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int64_t t = key_token(tile, n_routed_tiles, n_groups, s_groups, own_start, 4 * ty + a);
            if (t < T_hist) continue;                 // padding (-1) or detached history
            float* dkr = dKh + (t - T_hist) * D;
            float* dvr = dVh + (t - T_hist) * D;
#pragma unroll
            for (int j = 0; j < NC; ++j) {
                atomicAdd(dkr + tx + 16 * j, dk[a][j] * scale);
                atomicAdd(dvr + tx + 16 * j, dv[a][j]);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int j = 0; j < NC; ++j) dQ[(row0 + 4 * ty + a) * D + tx + 16 * j] = dq[a][j] * scale;
}

template <int D> constexpr size_t fwd_smem(int wg)
{
    return sizeof(float) * (3 * kTile * padded<D>() + kTile * (kTile + 1)) + sizeof(int) * wg;
}
template <int D> constexpr size_t bwd_smem(int wg)
{
    return sizeof(float) * (4 * kTile * padded<D>() + 2 * kTile * (kTile + 1)) + sizeof(int) * wg;
}

template <typename TIn, int D>
cudaError_t launch_fwd(const Shape& s, const void* Q, const void* K, const void* V,
                       const int32_t* gidx, float* O, float* lse, cudaStream_t st)
{
    const size_t smem = fwd_smem<D>(s.wg);
    auto k = attn_fwd_simt_kernel<TIn, D>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (int64_t)s.B * s.Hq * s.nQB;
    k<<<(unsigned)blocks, kThreads, smem, st>>>(
        static_cast<const TIn*>(Q), static_cast<const TIn*>(K), static_cast<const TIn*>(V), gidx, O,
        lse, s.Hq, s.Hkv, s.G, s.T_hist, s.T_seg, s.nQB, s.cap, s.wg, s.scale * kLog2e);
    return cudaGetLastError();
}

template <typename TIn, int D>
cudaError_t launch_bwd(const Shape& s, const void* Q, const void* K, const void* V, const float* O,
                       const float* lse, const void* dO, const int32_t* gidx, float* dQ,
                       float* dK_seg, float* dV_seg, float* Drow, cudaStream_t st)
{
    const int64_t rows = (int64_t)s.B * s.Hq * s.T_seg;
    bwd_rowdot_kernel<TIn, D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
        O, static_cast<const TIn*>(dO), Drow, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t seg_bytes = sizeof(float) * (size_t)s.B * s.Hkv * s.T_seg * s.d;
    if ((e = cudaMemsetAsync(dK_seg, 0, seg_bytes, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dV_seg, 0, seg_bytes, st)) != cudaSuccess) return e;
    const size_t smem = bwd_smem<D>(s.wg);
    auto k = attn_bwd_simt_kernel<TIn, D>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return e;
    const int64_t blocks = (int64_t)s.B * s.Hq * s.nQB;
    k<<<(unsigned)blocks, kThreads, smem, st>>>(
        static_cast<const TIn*>(Q), static_cast<const TIn*>(K), static_cast<const TIn*>(V), lse,
        static_cast<const TIn*>(dO), Drow, gidx, dQ, dK_seg, dV_seg, s.Hq, s.Hkv, s.G, s.T_hist,
        s.T_seg, s.nQB, s.cap, s.wg, s.scale, s.scale * kLog2e);
    return cudaGetLastError();
}

}  // namespace

size_t attn_simt_smem(const Shape& s, bool backward)
{
    if (s.d == 128) return backward ? bwd_smem<128>(s.wg) : fwd_smem<128>(s.wg);
    return backward ? bwd_smem<64>(s.wg) : fwd_smem<64>(s.wg);
}

cudaError_t launch_attn_fwd_simt(const Shape& s, const void* Q, const void* K, const void* V,
                                 const int32_t* gidx, float* O, float* lse, cudaStream_t st)
{
    if (s.dtype == HGA_BF16)
        return s.d == 128 ? launch_fwd<__nv_bfloat16, 128>(s, Q, K, V, gidx, O, lse, st)
                          : launch_fwd<__nv_bfloat16, 64>(s, Q, K, V, gidx, O, lse, st);
    return s.d == 128 ? launch_fwd<float, 128>(s, Q, K, V, gidx, O, lse, st)
                      : launch_fwd<float, 64>(s, Q, K, V, gidx, O, lse, st);
}

cudaError_t launch_attn_bwd_simt(const Shape& s, const void* Q, const void* K, const void* V,
                                 const float* O, const float* lse, const void* dO,
                                 const int32_t* gidx, float* dQ, float* dK_seg, float* dV_seg,
                                 float* Drow, cudaStream_t st)
{
    if (s.dtype == HGA_BF16)
        return s.d == 128 ? launch_bwd<__nv_bfloat16, 128>(s, Q, K, V, O, lse, dO, gidx, dQ, dK_seg,
                                                           dV_seg, Drow, st)
                          : launch_bwd<__nv_bfloat16, 64>(s, Q, K, V, O, lse, dO, gidx, dQ, dK_seg,
                                                          dV_seg, Drow, st);
    return s.d == 128 ? launch_bwd<float, 128>(s, Q, K, V, O, lse, dO, gidx, dQ, dK_seg, dV_seg,
                                               Drow, st)
                      : launch_bwd<float, 64>(s, Q, K, V, O, lse, dO, gidx, dQ, dK_seg, dV_seg,
                                              Drow, st);
}

// Check word of this translation unit's bounds checks (checked builds).
HGA_CHECK_WORD_READER(check_word_attn_simt)

}  // namespace hga
