// selftest.cu -- exercises the library's failure path on the device: a
// bounded mbarrier wait that runs out.
//
// Every tensor-core and decode kernel waits on mbarriers with a time limit;
// when a wait runs out, the kernel records the wait's code in a device
// status word, winds down (frees its tensor memory) and returns instead of
// hanging the GPU, and the host reads the word with hga_device_status.
// hga_selftest_wait runs that path on purpose: one CTA allocates tensor
// memory, waits with a caller-given limit on an mbarrier that nothing ever
// arrives at, records kSiteSelftest, releases the tensor memory and
// returns.  No fault, trap or unbounded wait is involved.
#include "hga_internal.cuh"
#include "sm100.cuh"

namespace hga {
namespace {

using namespace sm100;

constexpr int kSiteSelftest = 901;

__global__ void __launch_bounds__(64, 1) selftest_wait_kernel(unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t slot;
    const int warp = threadIdx.x / 32;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(smem_u32(&slot), 32);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // Nothing arrives on `bar`: the wait gives up after limit_ns.
    if (threadIdx.x == 0) mbar_wait_limit(smem_u32(&bar), 0, kSiteSelftest, limit_ns);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(slot, 32);
    }
}

}  // namespace

int selftest_site() { return kSiteSelftest; }

cudaError_t launch_selftest_wait(unsigned long long limit_ns, cudaStream_t st)
{
    selftest_wait_kernel<<<1, 64, 0, st>>>(limit_ns);
    return cudaGetLastError();
}

int selftest_status(bool clear)
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
