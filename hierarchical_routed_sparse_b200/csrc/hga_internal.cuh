// hga_internal.cuh -- device helpers and kernel launchers shared by the
// translation units of libhga.so.  Not part of the public ABI.
#pragma once
#include <atomic>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hga.h"

namespace hga {

constexpr int kChunk = 64;   // tokens per chunk == queries per block
constexpr int kGroup = 8;    // tokens per group
constexpr int kGroupsPerChunk = kChunk / kGroup;

// Validated problem shape handed to every launcher.
struct Shape {
    int B, Hq, Hkv, G, d;
    int64_t T_hist, T_seg, T;
    int64_t nC, nG, nQB;     // chunks, groups (whole context), query blocks
    int64_t cap;             // K / V rows per (batch, kv-head) (row stride of K, V)
    int64_t nCs, nGs;        // row strides of csum / gsum per (batch, kv-head): cap / 64, cap / 8
    int k_c, k_g;            // <= 0: keep all eligible
    int wc, wg;              // index row widths
    float scale;
    int dtype;
};

// Work items of the tensor-core backward: one per (batch, kv-head, query
// block) and pair of q-heads.  At most B*Hq*T_seg / 64.
inline int64_t bwd_items(const Shape& s) { return (int64_t)s.B * s.Hkv * s.nQB * ((s.G + 1) / 2); }

// Backward scratch, in floats: the row sums D (B*Hq*T_seg floats), then the
// backward's item schedule (one int32 per item).
inline int64_t bwd_scratch_floats(const Shape& s) { return (int64_t)s.B * s.Hq * s.T_seg + bwd_items(s); }

// ---- element loads --------------------------------------------------------
// 16-byte vector of inputs widened to float32 (8 bf16 or 4 float).
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int E = 8;
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* out) {
        const uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <> struct Vec16<float> {
    static constexpr int E = 4;
    static __device__ __forceinline__ void load(const float* p, float* out) {
        const float4 r = __ldg(reinterpret_cast<const float4*>(p));
        out[0] = r.x; out[1] = r.y; out[2] = r.z; out[3] = r.w;
    }
};

// ---- routing keys -----------------------------------------------------------
// A candidate (score, index) packed so that a larger 64-bit key means a higher
// score, and among equal scores the lower index.  -0.0 is folded into +0.0 so
// that the two compare equal, as they do in floating point.
__device__ __forceinline__ unsigned long long pack_key(float s, int32_t idx) {
    uint32_t u = __float_as_uint(s + 0.0f);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (static_cast<unsigned long long>(u) << 32) | static_cast<uint32_t>(~idx);
}
__device__ __forceinline__ int32_t key_index(unsigned long long k) {
    return static_cast<int32_t>(~static_cast<uint32_t>(k & 0xFFFFFFFFull));
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long w = __shfl_xor_sync(0xFFFFFFFFu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// ---- programmatic dependent launch ------------------------------------------------
// The library's kernels are launched so that each may start while the kernel
// before it on the stream finishes (its launch and setup overlap that
// kernel's last CTAs).  A kernel calls pdl_wait() before its first access to
// global memory -- the previous kernel, the library's or the caller's, may be
// writing any of its inputs -- and pdl_trigger() right after, which lets the
// next kernel launch.  Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Raise a kernel's dynamic shared memory limit to at least `bytes`, calling
// the driver only when the limit set so far (per kernel function and device)
// is lower: a repeated launch path makes no driver call besides the launch.
// Kernels of one signature (template instances that differ only in
// compile-time parameters) are told apart by their address (tma_map.cu).
cudaError_t allow_smem_fn(const void* kernel, int bytes);
template <typename Kern>
cudaError_t allow_smem(Kern kernel, int bytes)
{
    return allow_smem_fn(reinterpret_cast<const void*>(kernel), bytes);
}

// ---- launchers (each returns cudaError_t of its launch) ------------------------
// K holds T_src rows per (batch, kv-head), the first of them at position row0.
cudaError_t launch_summaries(const Shape& s, const void* K, int64_t T_src, int64_t row0, int64_t c_begin,
                             int64_t c_end, float* csum, float* gsum, cudaStream_t st);
cudaError_t launch_route_chunks(const Shape& s, const void* Q, const float* csum, float* qbar,
                                int32_t* cidx, cudaStream_t st);
cudaError_t launch_route_groups(const Shape& s, const float* qbar, const float* gsum,
                                const int32_t* cidx, int32_t* gidx, cudaStream_t st);
cudaError_t launch_route_fused(const Shape& s, const void* Q, const float* csum, const float* gsum,
                               float* qbar, int32_t* cidx, int32_t* gidx, cudaStream_t st);
size_t route_fused_smem(const Shape& s);
// One decode step of the token at position pos (decode.cu).
cudaError_t launch_decode(const Shape& s, int64_t pos, const void* q, const void* K, const void* V,
                          const float* csum, const float* gsum, float* O, float* lse, int32_t* cidx,
                          int32_t* gidx, cudaStream_t st);
size_t decode_smem(const Shape& s);
int decode_max_heads();
int decode_status(bool clear);   // status word of decode.cu's bounded waits
// Check words of the bounds checks (checked builds; 0 otherwise), one per
// translation unit that reads caller index rows.
int check_word_attn_tc_fwd(bool clear);
int check_word_attn_tc_bwd(bool clear);
int check_word_attn_simt(bool clear);
int check_word_causal(bool clear);
int check_word_router(bool clear);
int check_word_stage(bool clear);
int selftest_status(bool clear); // status word of selftest.cu
int selftest_site();             // the code its wait records
cudaError_t launch_selftest_wait(unsigned long long limit_ns, cudaStream_t st);
// Strictly causal variant: routing per query position (causal.cu).
cudaError_t launch_route_causal(const Shape& s, const void* Q, const float* csum, const float* gsum, int32_t* cidx,
                                int32_t* gidx, cudaStream_t st);
// sched: the order of the tensor-core kernels' window items (CTA x runs item
// sched[x]), or null for index order; the warp-per-row kernels ignore it.
cudaError_t launch_attn_fwd_causal(const Shape& s, const void* Q, const void* K, const void* V, const int32_t* gidx,
                                   const int32_t* sched, float* O, float* lse, cudaStream_t st);
cudaError_t launch_attn_bwd_causal(const Shape& s, const void* Q, const void* K, const void* V, const float* O,
                                   const float* lse, const void* dO, const int32_t* gidx, const int32_t* sched,
                                   float* dQ, float* dK, float* dV, cudaStream_t st);
size_t route_causal_smem(const Shape& s);
int causal_max_heads();
// Window items of the causal tensor-core kernels (B * Hkv * windows * head
// quads), the schedule kernel's shared memory, and the schedule itself:
// sched[0, n) the items heaviest first, sched[n, 2n) their costs.
int64_t causal_items(const Shape& s);
size_t causal_sched_smem(const Shape& s);
cudaError_t launch_causal_schedule(const Shape& s, const int32_t* gidx, int32_t* sched, cudaStream_t st);
cudaError_t launch_attn_fwd_simt(const Shape& s, const void* Q, const void* K, const void* V,
                                 const int32_t* gidx, float* O, float* lse, cudaStream_t st);
cudaError_t launch_attn_bwd_simt(const Shape& s, const void* Q, const void* K, const void* V,
                                 const float* O, const float* lse, const void* dO,
                                 const int32_t* gidx, float* dQ, float* dK_seg, float* dV_seg,
                                 float* Drow, cudaStream_t st);

// Streaming multiprocessors of the current device (cached per device).
int sm_count();

// TMA tensor maps (tma_map.cu).
bool tensor_maps_available();
bool make_bf16_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
bool make_f32_map(CUtensorMap* map, void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

// Tensor-core (tcgen05) path for bf16 inputs.
bool attn_fwd_tc_supported(const Shape& s);
cudaError_t launch_attn_fwd_tc(const Shape& s, const void* Q, const void* K, const void* V,
                               const int32_t* gidx, float* O, float* lse, cudaStream_t st);
// Status word of the tensor-core kernels' bounded waits (0 = none ran out;
// -1 = could not be read).  Synchronises with the device.
int attn_fwd_tc_status(bool clear);
bool route_attn_fwd_tc_supported(const Shape& s);
cudaError_t launch_route_attn_fwd_tc(const Shape& s, const void* Q, const void* K, const void* V, const float* csum,
                                     const float* gsum, float* qbar, int32_t* cidx, int32_t* gidx, float* O,
                                     float* lse, cudaStream_t st);
bool attn_fwd_tc_causal_supported(const Shape& s);
cudaError_t launch_attn_fwd_tc_causal(const Shape& s, const void* Q, const void* K, const void* V,
                                      const int32_t* gidx, const int32_t* sched, float* O, float* lse,
                                      cudaStream_t st);
bool attn_bwd_tc_supported(const Shape& s);
cudaError_t launch_attn_bwd_tc(const Shape& s, const void* Q, const void* K, const void* V,
                               const float* O, const float* lse, const void* dO,
                               const int32_t* gidx, float* dQ, float* dK_seg, float* dV_seg,
                               float* Drow, cudaStream_t st);
int attn_bwd_tc_status(bool clear);
bool attn_bwd_tc_causal_supported(const Shape& s);
cudaError_t launch_attn_bwd_tc_causal(const Shape& s, const void* Q, const void* K, const void* V, const float* O,
                                      const float* lse, const void* dO, const int32_t* gidx,
                                      const int32_t* sched, float* dQ, float* dK_seg, float* dV_seg,
                                      cudaStream_t st);

}  // namespace hga
