// stage.cu -- host-RAM KV tier: gather the routed history groups into a
// device staging buffer.
//
// Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com):
// older KV can live in host RAM, and after routing only the selected groups'
// exact tokens are brought to the GPU for the attention (sections "What HGA
// does differently" and "How it fits in 16 GB").  Here history K/V rows may
// sit in pinned, device-mapped host memory; after routing, every routed
// history group is copied (plain 16-byte loads, no TMA) into a staging
// buffer in HBM, the segment's own rows are appended, and the index rows are
// rewritten so that the unchanged attention kernels run on the staged copy.
//
// Staged layout per (batch, kv-head): T_stage = round64(nQB * wg * 8)
// history rows -- slot j of query block qb holds the 8 rows of that block's
// j-th routed group at rows (qb*wg + j)*8 -- then the T_seg segment rows.
// A routed history group j maps to staged group qb*wg + slot, a segment
// group to T_stage/8 + (j - T_hist/8); padding stays -1.  Every row stays
// ascending with history before segment, and the segment keys keep their
// offsets past the history, so the backward's dK_seg / dV_seg are unchanged.
#include "hga_internal.cuh"

namespace hga {
namespace {

// One warp per (item u, slot j).  el_bytes = element size; row_bytes = d*el.
__global__ void __launch_bounds__(256)
stage_groups_kernel(const uint8_t* __restrict__ Kh, const uint8_t* __restrict__ Vh,
                    const int32_t* __restrict__ gidx, uint8_t* __restrict__ Ks, uint8_t* __restrict__ Vs,
                    int32_t* __restrict__ gidx_s, int64_t n_slots, int wg, int64_t nQB, int64_t T_hist,
                    int64_t T_stage, int64_t T_seg, int row_bytes)
{
    pdl_wait();
    pdl_trigger();
    const int64_t slot = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (slot >= n_slots) return;
    const int64_t u = slot / wg;                     // (b*Hkv + g)*nQB + qb
    const int j = int(slot % wg);
    const int64_t qb = u % nQB, bg = u / nQB;
    const int32_t grp = __ldg(gidx + slot);
    const int64_t first_seg_group = T_hist / 8;
    int32_t out;
    if (grp < 0) {
        out = -1;
    } else if (grp >= first_seg_group) {
        out = int32_t(T_stage / 8 + (grp - first_seg_group));
    } else {
        out = int32_t(qb * wg + j);
        // 8 rows of K and of V, 16 bytes per lane per step.
        const int64_t src = (bg * T_hist + (int64_t)grp * 8) * row_bytes;
        const int64_t dst = (bg * (T_stage + T_seg) + (int64_t)out * 8) * row_bytes;
        const int n16 = 8 * row_bytes / 16;
        for (int i = lane; i < n16; i += 32) {
            const uint4 k = *reinterpret_cast<const uint4*>(Kh + src + 16 * (int64_t)i);
            const uint4 v = *reinterpret_cast<const uint4*>(Vh + src + 16 * (int64_t)i);
            *reinterpret_cast<uint4*>(Ks + dst + 16 * (int64_t)i) = k;
            *reinterpret_cast<uint4*>(Vs + dst + 16 * (int64_t)i) = v;
        }
    }
    if (lane == 0) gidx_s[slot] = out;
}

}  // namespace

int64_t stage_hist_rows(const Shape& s)
{
    const int64_t rows = s.nQB * (int64_t)s.wg * 8;
    return (rows + 63) / 64 * 64;
}

cudaError_t launch_stage(const Shape& s, const void* K_hist, const void* V_hist, const void* K_seg,
                         const void* V_seg, const int32_t* gidx, void* K_stage, void* V_stage,
                         int32_t* gidx_stage, cudaStream_t st)
{
    const int el = s.dtype == HGA_BF16 ? 2 : 4;
    const int row_bytes = s.d * el;
    const int64_t T_stage = stage_hist_rows(s);
    const int64_t n_slots = (int64_t)s.B * s.Hkv * s.nQB * s.wg;
    if (n_slots > 0) {
        cudaError_t e = launch_pdl(stage_groups_kernel, dim3((unsigned)((n_slots + 7) / 8)), dim3(256), 0, st,
                                   static_cast<const uint8_t*>(K_hist), static_cast<const uint8_t*>(V_hist), gidx,
                                   static_cast<uint8_t*>(K_stage), static_cast<uint8_t*>(V_stage), gidx_stage,
                                   n_slots, s.wg, s.nQB, s.T_hist, T_stage, s.T_seg, row_bytes);
        if (e != cudaSuccess) return e;
    }
    // The segment's own rows after the staged history of each (batch, kv-head).
    const size_t seg_bytes = (size_t)s.T_seg * row_bytes;
    const size_t dst_pitch = (size_t)(T_stage + s.T_seg) * row_bytes;
    const size_t height = (size_t)s.B * s.Hkv;
    if (seg_bytes == 0) return cudaSuccess;
    for (int w = 0; w < 2; ++w) {
        uint8_t* dst = static_cast<uint8_t*>(w == 0 ? K_stage : V_stage) + (size_t)T_stage * row_bytes;
        const void* src = w == 0 ? K_seg : V_seg;
        cudaError_t e = cudaMemcpy2DAsync(dst, dst_pitch, src, seg_bytes, seg_bytes, height,
                                          cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace hga
