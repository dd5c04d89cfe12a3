// check.cuh -- bounds checks of the HGA_CHECK_BOUNDS build on the index rows
// that callers hand to the library.
//
// The attention, staging and group-routing calls read routed group (or
// chunk) indices from caller-provided rows and turn them into addresses.  A
// valid index lies in [0, limit): group indices before the row's own chunk
// (8 * own chunk), chunk indices before it (own chunk).  In a build compiled
// with -DHGA_CHECK_BOUNDS every such index is checked before it is used: an
// index outside records a site code in the translation unit's check word
// and is replaced by index 0 of the same (batch, kv-head), so the access
// that follows stays inside the tensors (the outputs are then invalid and
// the call reports HGA_ERR_DEVICE_CHECK).  A check never traps.  Release
// builds compile the checks away.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace hga {
namespace chk {

// Check word of the including translation unit: 0, or the site code of the
// first failed check.
static __device__ int g_check = 0;

#ifdef HGA_CHECK_BOUNDS
constexpr bool kEnabled = true;
#else
constexpr bool kEnabled = false;
#endif

// Site codes (which kernel and which read).
enum : int {
    kSiteFwdTc = 401, kSiteBwdTcLoad, kSiteBwdTcKeys, kSiteSimtFwd, kSiteSimtBwd, kSiteCausalFwd,
    kSiteCausalBwd, kSiteRouteGroups, kSiteStage, kSiteCausalSched
};

__device__ __forceinline__ int32_t index(int32_t j, int64_t limit, int site)
{
    if (kEnabled && (j < 0 || (int64_t)j >= limit)) {
        atomicCAS(&g_check, 0, site);
        return 0;
    }
    return j;
}

// A group index of a routed row; `limit` = 8 * (own chunk).
__device__ __forceinline__ int32_t group(int32_t j, int64_t limit, int site) { return index(j, limit, site); }
// A chunk index of a routed row; `limit` = own chunk.
__device__ __forceinline__ int32_t chunk(int32_t c, int64_t limit, int site) { return index(c, limit, site); }

// Record `site` when `bad` (checked builds only).
__device__ __forceinline__ void flag_if(bool bad, int site)
{
    if (kEnabled && bad) atomicCAS(&g_check, 0, site);
}

// Item sched[x] of a caller's item order for CTA x of a one-item-per-CTA
// grid.  Checked in every build (one load per CTA): an entry outside
// [0, gridDim.x) is replaced by x, so no item index leaves the grid's range,
// and checked builds record it.
__device__ __forceinline__ int64_t sched_item(const int32_t* sched)
{
    const int64_t x = blockIdx.x;
    if (!sched) return x;
    const int32_t it = __ldg(sched + x);
    const bool bad = it < 0 || (uint32_t)it >= gridDim.x;
    flag_if(bad, kSiteCausalSched);
    return bad ? x : it;
}

}  // namespace chk
}  // namespace hga

// Defines `int fn(bool clear)`: the translation unit's check word (-1 if it
// could not be read), cleared when `clear`.  Synchronous.
#define HGA_CHECK_WORD_READER(fn)                                                           \
    int fn(bool clear)                                                                      \
    {                                                                                       \
        int v = 0;                                                                          \
        if (cudaMemcpyFromSymbol(&v, hga::chk::g_check, sizeof v) != cudaSuccess) return -1; \
        if (clear && v) {                                                                   \
            const int z = 0;                                                                \
            cudaMemcpyToSymbol(hga::chk::g_check, &z, sizeof z);                            \
        }                                                                                   \
        return v;                                                                           \
    }
