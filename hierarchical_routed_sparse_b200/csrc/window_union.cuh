// window_union.cuh -- the routed groups of a window of neighbouring query
// positions, merged (strictly causal variant).
//
// In the strictly causal variant every query position routes on its own
// query (article "BMW's 16 GB GPU just did what needs an A100", section
// "The one real caveat: causal leakage"), so each position has its own row
// of routed groups.  The tensor-core kernels process kWin neighbouring
// positions of one (batch, kv-head) together: their key tiles are the union
// of the kWin rows' groups, ascending, and a kWin-bit mask per union group
// names the positions that routed it, so every query row keeps only the keys
// of its own routing.  The union is built in shared memory by the whole CTA:
// a bitmap over the eligible groups, prefix counts of its words (the rank of
// a group in the union), then the list and the masks.
#pragma once

#include <stdint.h>

#include "check.cuh"

namespace hga {
namespace wu {

constexpr int kWin = 32;     // positions of a window (one bit each in a mask)

// Shared-memory bytes of the builder for at most `n_groups` eligible groups
// and index rows of width `wg`.
__host__ __device__ constexpr size_t bytes(int64_t n_groups, int wg)
{
    return 8 * (size_t)((n_groups + 31) / 32) + 8 * (size_t)kWin * (size_t)wg;
}

struct View {
    uint32_t* bitmap;    // [nwords_max]
    uint32_t* prefix;    // [nwords_max]
    int32_t* list;       // [kWin * wg] union groups, ascending
    uint32_t* mask;      // [kWin * wg] bit p: position p of the window routed list[k]
};

__device__ __forceinline__ View view(uint8_t* buf, int64_t n_groups, int wg)
{
    const int64_t nw = (n_groups + 31) / 32;
    View v;
    v.bitmap = reinterpret_cast<uint32_t*>(buf);
    v.prefix = v.bitmap + nw;
    v.list = reinterpret_cast<int32_t*>(v.prefix + nw);
    v.mask = reinterpret_cast<uint32_t*>(v.list + (size_t)kWin * wg);
    return v;
}

// Whole-CTA call.  rows: the kWin routing rows of the window, [kWin][wg]
// (ascending groups, -1 padded); valid groups lie in [0, limit), limit <=
// n_groups.  Entries outside are dropped, so no index outside the tensors
// is ever formed (checked builds also record them).
// Returns the number of union groups.
__device__ __forceinline__ int build(const int32_t* __restrict__ rows, int wg, int64_t limit, const View& v, int* s_n, int site)
{
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
    const int nwords = int((limit + 31) / 32);
    const int n_e = kWin * wg;
    for (int w = tid; w < nwords; w += nt) v.bitmap[w] = 0u;
    __syncthreads();
    for (int e = tid; e < n_e; e += nt) {
        const int32_t j = __ldg(rows + e);
        if (j < 0) continue;                          // padding
        chk::flag_if(j >= limit, site);
        if (j >= limit) continue;                     // not eligible: dropped, never addressed
        atomicOr(&v.bitmap[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    if (tid < 32) {                                   // exclusive prefix of the word popcounts
        int run = 0;
        for (int base = 0; base < nwords; base += 32) {
            const int w = base + lane;
            const int cnt = w < nwords ? __popc(v.bitmap[w]) : 0;
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += y;
            }
            if (w < nwords) v.prefix[w] = uint32_t(run + incl - cnt);
            run += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) *s_n = run;
    }
    __syncthreads();
    const int n = *s_n;
    for (int k = tid; k < n; k += nt) v.mask[k] = 0u;
    for (int w = tid; w < nwords; w += nt) {          // the list, ascending
        uint32_t word = v.bitmap[w];
        int k = int(v.prefix[w]);
        while (word) {
            const int b = __ffs(word) - 1;
            v.list[k++] = w * 32 + b;
            word &= word - 1;
        }
    }
    __syncthreads();
    for (int e = tid; e < n_e; e += nt) {
        const int32_t j = __ldg(rows + e);
        if (j < 0 || j >= limit) continue;            // as counted above
        const uint32_t word = v.bitmap[j >> 5];
        const int rank = int(v.prefix[j >> 5]) + __popc(word & ((1u << (j & 31)) - 1u));
        atomicOr(&v.mask[rank], 1u << (e / wg));
    }
    __syncthreads();
    return n;
}

}  // namespace wu
}  // namespace hga
