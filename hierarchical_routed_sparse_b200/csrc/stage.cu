// stage.cu -- host-RAM KV tier: gather the routed history groups into a
// device staging buffer.
//
// Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com):
// older KV can live in host RAM, and after routing only the selected groups'
// exact tokens are brought to the GPU for the attention (sections "What HGA
// does differently" and "How it fits in 16 GB").  Here history K/V rows may
// sit in pinned, device-mapped host memory; after routing, every history
// group routed by any query block is copied once (plain 16-byte loads, no
// TMA) into a staging buffer in HBM, the segment's own rows are appended,
// and the index rows are rewritten so that the unchanged attention kernels
// run on the staged copy.
//
// Staged layout per (batch, kv-head): T_stage = round64(nQB * wg * 8)
// history rows (room for every slot of every block); the n_u distinct routed
// history groups, in ascending group order, occupy rows 0 .. 8 n_u - 1 --
// group number k of that order at rows 8k .. 8k + 7 -- then come the T_seg
// segment rows.  A routed history group maps to its rank k among the
// distinct ones, a segment group j to T_stage/8 + (j - T_hist/8); padding
// stays -1.  The map is increasing, so every row stays ascending with
// history before segment, and the segment keys keep their offsets past the
// history, so the backward's dK_seg / dV_seg are unchanged.
#include "check.cuh"
#include "hga_internal.cuh"

namespace hga {
namespace {

constexpr int kStageCtas = 16;      // CTAs per (batch, kv-head)

// Grid: kStageCtas CTAs per (batch, kv-head) unit, 256 threads.  Every CTA
// of a unit builds the same plan in shared memory -- a bitmap of the
// history groups routed by any of the unit's query blocks and the exclusive
// prefix of its words' popcounts, so that the rank of a set group is
// pre[w] + popc(bits below it) -- then rewrites its share of the unit's
// index rows and copies its share of the set groups (warp x of CTA c takes
// groups x + 8 c, stepping by 8 kStageCtas), 8 rows of K and of V per
// group with every lane's 16-byte loads in flight before its stores.
__global__ void __launch_bounds__(256)
stage_unique_kernel(const uint8_t* __restrict__ Kh, const uint8_t* __restrict__ Vh,
                    const int32_t* __restrict__ gidx, uint8_t* __restrict__ Ks, uint8_t* __restrict__ Vs,
                    int32_t* __restrict__ gidx_s, int64_t nQB, int wg, int64_t T_hist, int64_t T_stage,
                    int64_t T_seg, int row_bytes)
{
    extern __shared__ uint32_t bm[];                 // [nwords] bits, then [nwords] prefix
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bg = blockIdx.x / kStageCtas;
    const int c = int(blockIdx.x % kStageCtas);
    const int64_t ng_hist = T_hist / 8;
    const int nwords = int((ng_hist + 31) / 32);
    uint32_t* pre = bm + nwords;
    const int64_t n = nQB * (int64_t)wg;
    const int32_t* gu = gidx + bg * n;
    for (int w = tid; w < nwords; w += 256) bm[w] = 0u;
    __syncthreads();
    for (int64_t e = tid; e < n; e += 256) {
        const int32_t g = __ldg(gu + e);
        if (g >= 0 && g < ng_hist) atomicOr(&bm[g >> 5], 1u << (g & 31));
    }
    __syncthreads();
    if (warp == 0) {                                 // exclusive prefix of the popcounts
        int run = 0;
        for (int base = 0; base < nwords; base += 32) {
            const int w = base + lane;
            const int cnt = w < nwords ? __popc(bm[w]) : 0;
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += y;
            }
            if (w < nwords) pre[w] = uint32_t(run + incl - cnt);
            run += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
    }
    __syncthreads();
    // This CTA's share of the index rows.
    for (int64_t e = (int64_t)c * 256 + tid; e < n; e += (int64_t)kStageCtas * 256) {
        const int32_t g = __ldg(gu + e);
        int32_t out;
        if (g < 0) {
            out = -1;
        } else if (g >= ng_hist) {
            // A segment group: in the staged problem it follows the T_stage
            // history rows.  Valid groups lie before the row's own chunk.
            chk::flag_if(g >= ng_hist + T_seg / 8, chk::kSiteStage);
            out = int32_t(T_stage / 8 + (g - ng_hist));
        } else {
            const uint32_t word = bm[g >> 5];
            out = int32_t(pre[g >> 5] + __popc(word & ((1u << (g & 31)) - 1u)));
        }
        gidx_s[bg * n + e] = out;
    }
    // This CTA's share of the copies.
    const int64_t row_stride = T_stage + T_seg;
    const int n16 = 8 * row_bytes / 16;              // 16-byte pieces of a group (<= 256)
    for (int64_t g = warp + 8 * (int64_t)c; g < ng_hist; g += 8 * (int64_t)kStageCtas) {
        const uint32_t word = bm[g >> 5];
        if (!((word >> (g & 31)) & 1u)) continue;
        const int64_t slot = pre[g >> 5] + __popc(word & ((1u << (g & 31)) - 1u));
        const int64_t src = (bg * T_hist + g * 8) * row_bytes;
        const int64_t dst = (bg * row_stride + slot * 8) * row_bytes;
        constexpr int kPer = 8;                      // pieces per lane in flight (n16 <= 256)
        uint4 kv[kPer], vv[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int piece = lane + 32 * q;
            if (piece < n16) {
                kv[q] = *reinterpret_cast<const uint4*>(Kh + src + 16 * (int64_t)piece);
                vv[q] = *reinterpret_cast<const uint4*>(Vh + src + 16 * (int64_t)piece);
            }
        }
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int piece = lane + 32 * q;
            if (piece < n16) {
                *reinterpret_cast<uint4*>(Ks + dst + 16 * (int64_t)piece) = kv[q];
                *reinterpret_cast<uint4*>(Vs + dst + 16 * (int64_t)piece) = vv[q];
            }
        }
    }
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
        const int nwords = int((s.T_hist / 8 + 31) / 32);
        const size_t smem = 2 * sizeof(uint32_t) * (size_t)(nwords > 0 ? nwords : 1);
        cudaError_t e = allow_smem(stage_unique_kernel, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(stage_unique_kernel, dim3((unsigned)(s.B * s.Hkv * kStageCtas)), dim3(256), smem, st,
                       static_cast<const uint8_t*>(K_hist), static_cast<const uint8_t*>(V_hist), gidx,
                       static_cast<uint8_t*>(K_stage), static_cast<uint8_t*>(V_stage), gidx_stage, s.nQB, s.wg,
                       s.T_hist, T_stage, s.T_seg, row_bytes);
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

// Check word of this translation unit's bounds checks (checked builds).
HGA_CHECK_WORD_READER(check_word_stage)

}  // namespace hga
