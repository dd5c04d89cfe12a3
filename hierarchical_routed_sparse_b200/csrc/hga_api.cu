// hga_api.cu -- the C ABI of libhga.so (declared in include/hga.h).
//
// Every entry point validates its arguments on the host, turns them into a
// hga::Shape and enqueues kernels on the caller's stream.  Nothing here
// allocates device memory or synchronises.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "hga_internal.cuh"

namespace hga {
size_t route_chunks_smem(const Shape& s);
size_t route_groups_smem(const Shape& s);
size_t attn_simt_smem(const Shape& s, bool backward);
}

namespace {

thread_local char g_err[512] = "";

// An NVTX range around one ABI call, named after it: profilers (ncu --nvtx,
// Nsight Systems) show the call and can select its kernels by the range.
// Without a tool attached a push / pop is a test of a null function pointer.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

int fail(int code, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char* where)
{
    return fail(HGA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

constexpr size_t kMaxSmem = 227 * 1024;

// First nonzero check word of the translation units that read caller index
// rows (-1 if one could not be read); cleared when `clear`.
int read_check_words(bool clear)
{
    int (*const readers[])(bool) = {hga::check_word_attn_tc_fwd, hga::check_word_attn_tc_bwd,
                                    hga::check_word_attn_simt,   hga::check_word_causal,
                                    hga::check_word_router,      hga::check_word_stage};
    int first = 0;
    for (auto f : readers) {
        const int v = f(clear);
        if (v < 0) return -1;
        if (!first) first = v;
    }
    return first;
}

// Result of a call that enqueued its kernels with launch status `e`.  In a
// build with HGA_CHECK_BOUNDS the call waits for its stream and reports a
// failed device bounds check as HGA_ERR_DEVICE_CHECK (the word is cleared);
// release builds return at once.
int finish(cudaError_t e, cudaStream_t st, const char* name)
{
    if (e != cudaSuccess) return cuda_fail(e, name);
#ifdef HGA_CHECK_BOUNDS
    e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, name);
    const int w = read_check_words(true);
    if (w < 0) return fail(HGA_ERR_CUDA, "%s: the bounds-check word could not be read", name);
    if (w)
        return fail(HGA_ERR_DEVICE_CHECK,
                    "%s: device bounds check %d failed: an index row holds an entry outside its valid range "
                    "(outputs are invalid)", name, w);
#else
    (void)st;
#endif
    return HGA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define CHECK_PTR(ptr)                                                                   \
    do {                                                                                 \
        if ((ptr) == nullptr) return fail(HGA_ERR_INVALID_ARG, "%s is NULL", #ptr);      \
        if (!aligned16(ptr)) return fail(HGA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #ptr); \
    } while (0)

// Validate the parameter block and derive the shape.  Returns HGA_OK or an
// error code with the message set.
int make_shape(const hga_params* p, hga::Shape* s)
{
    if (!p) return fail(HGA_ERR_INVALID_ARG, "params is NULL");
    if (p->B < 1 || p->Hq < 1 || p->Hkv < 1)
        return fail(HGA_ERR_INVALID_ARG, "B, Hq, Hkv must be >= 1 (got %d, %d, %d)", p->B, p->Hq, p->Hkv);
    if (p->Hq % p->Hkv != 0)
        return fail(HGA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", p->Hq, p->Hkv);
    if (p->d != 64 && p->d != 128) return fail(HGA_ERR_UNSUPPORTED, "head dim d=%d (supported: 64, 128)", p->d);
    if (p->chunk != hga::kChunk || p->group != hga::kGroup || p->qblock != hga::kChunk)
        return fail(HGA_ERR_UNSUPPORTED, "chunk/group/qblock must be 64/8/64 (got %d/%d/%d)", p->chunk,
                    p->group, p->qblock);
    if (p->T_hist < 0 || p->T_seg < 0 || p->T_hist % 64 || p->T_seg % 64)
        return fail(HGA_ERR_INVALID_ARG, "T_hist (%lld) and T_seg (%lld) must be non-negative multiples of 64",
                    (long long)p->T_hist, (long long)p->T_seg);
    if ((p->k_c < 1 && p->k_c != HGA_ALL) || (p->k_g < 1 && p->k_g != HGA_ALL))
        return fail(HGA_ERR_INVALID_ARG, "k_c (%d) and k_g (%d) must be >= 1 or HGA_ALL", p->k_c, p->k_g);
    if (p->dtype != HGA_BF16 && p->dtype != HGA_FP32)
        return fail(HGA_ERR_INVALID_ARG, "dtype %d is neither HGA_BF16 nor HGA_FP32", p->dtype);
    if (!std::isfinite(p->scale) || p->scale < 0.f)
        return fail(HGA_ERR_INVALID_ARG, "scale must be finite and >= 0 (0 selects 1/sqrt(d))");
    const int64_t T = p->T_hist + p->T_seg;
    if (T / hga::kGroup > INT32_MAX)
        return fail(HGA_ERR_UNSUPPORTED, "context of %lld tokens overflows int32 group indices", (long long)T);
    s->B = p->B; s->Hq = p->Hq; s->Hkv = p->Hkv; s->G = p->Hq / p->Hkv; s->d = p->d;
    s->T_hist = p->T_hist; s->T_seg = p->T_seg; s->T = T;
    s->nC = T / hga::kChunk; s->nG = T / hga::kGroup; s->nQB = p->T_seg / hga::kChunk;
    if (p->kv_capacity != 0 && (p->kv_capacity < T || p->kv_capacity % 64))
        return fail(HGA_ERR_INVALID_ARG, "kv_capacity (%lld) must be 0 or a multiple of 64 >= T_hist + T_seg (%lld)",
                    (long long)p->kv_capacity, (long long)T);
    s->cap = p->kv_capacity ? p->kv_capacity : T;
    if (s->cap / hga::kGroup > INT32_MAX)
        return fail(HGA_ERR_UNSUPPORTED, "kv_capacity of %lld rows overflows int32 group indices", (long long)s->cap);
    s->nCs = s->cap / hga::kChunk; s->nGs = s->cap / hga::kGroup;
    s->k_c = p->k_c == HGA_ALL ? 0 : p->k_c;
    s->k_g = p->k_g == HGA_ALL ? 0 : p->k_g;
    const int64_t wc = p->k_c == HGA_ALL ? (s->nC > 0 ? s->nC : 1) : p->k_c;
    const int64_t wg = p->k_g == HGA_ALL ? wc * hga::kGroupsPerChunk : p->k_g;
    if (wc > INT32_MAX / 64 || wg > INT32_MAX / 64)
        return fail(HGA_ERR_UNSUPPORTED, "routing widths too large (wc=%lld, wg=%lld)", (long long)wc,
                    (long long)wg);
    s->wc = (int)wc; s->wg = (int)wg;
    s->scale = p->scale == 0.f ? 1.0f / std::sqrt((float)p->d) : p->scale;
    s->dtype = p->dtype;
    const int64_t units = (int64_t)s->B * s->Hq * (s->nQB > 0 ? s->nQB : 1);
    if (units > INT32_MAX || (int64_t)s->B * s->Hkv * (s->nC > 0 ? s->nC : 1) > INT32_MAX)
        return fail(HGA_ERR_UNSUPPORTED, "problem too large for one launch grid");
    return HGA_OK;
}


// The backward kernels: bf16 with d = 128 on the tensor cores, everything
// else on the FMA kernel.  Drow is the scratch of hga::bwd_scratch_floats:
// row sums, then (tensor-core kernel only) the item schedule.
cudaError_t run_attn_bwd(const hga::Shape& s, const void* Q, const void* K, const void* V, const float* O,
                         const float* lse, const void* dO, const int32_t* gidx, float* dQ, float* dK_seg,
                         float* dV_seg, float* Drow, cudaStream_t st)
{
    if (hga::attn_bwd_tc_supported(s))
        return hga::launch_attn_bwd_tc(s, Q, K, V, O, lse, dO, gidx, dQ, dK_seg, dV_seg, Drow, st);
    return hga::launch_attn_bwd_simt(s, Q, K, V, O, lse, dO, gidx, dQ, dK_seg, dV_seg, Drow, st);
}

// A pointer the device can load from: device (or managed) memory as it is,
// device-mapped host memory by its device address; pageable host memory is
// refused.
int device_addressable(const void* ptr, const void** dev, const char* name)
{
    cudaPointerAttributes at;
    const cudaError_t e = cudaPointerGetAttributes(&at, ptr);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(HGA_ERR_INVALID_ARG, "%s: the pointer is unknown to CUDA (%s)", name, cudaGetErrorName(e));
    }
    if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) {
        *dev = ptr;
        return HGA_OK;
    }
    if (at.type == cudaMemoryTypeHost && at.devicePointer != nullptr) {
        *dev = at.devicePointer;
        return HGA_OK;
    }
    return fail(HGA_ERR_INVALID_ARG, "%s: host memory the device cannot address (pin and map it)", name);
}

}  // namespace

namespace hga {
int64_t stage_hist_rows(const Shape& s);
cudaError_t launch_stage(const Shape& s, const void* K_hist, const void* V_hist, const void* K_seg,
                         const void* V_seg, const int32_t* gidx, void* K_stage, void* V_stage,
                         int32_t* gidx_stage, cudaStream_t st);
}

extern "C" {

const char* hga_last_error(void) { return g_err; }

const char* hga_version(void) { return "hga-b200 0.1 (sm_100a)"; }

int hga_device_status(int* status, int clear)
{
    const NvtxRange nvtx_range("hga_device_status");
    if (!status) return fail(HGA_ERR_INVALID_ARG, "status is NULL");
    const int vf = hga::attn_fwd_tc_status(clear != 0);
    const int vb = hga::attn_bwd_tc_status(clear != 0);
    const int vd = hga::decode_status(clear != 0);
    const int vs = hga::selftest_status(clear != 0);
    if (vf < 0 || vb < 0 || vd < 0 || vs < 0)
        return fail(HGA_ERR_CUDA, "hga_device_status: the status word could not be read");
    *status = vf ? vf : (vb ? vb : (vd ? vd : vs));
    return HGA_OK;
}

int hga_device_check(int* word, int clear)
{
    const NvtxRange nvtx_range("hga_device_check");
    if (!word) return fail(HGA_ERR_INVALID_ARG, "word is NULL");
    const int w = read_check_words(clear != 0);
    if (w < 0) return fail(HGA_ERR_CUDA, "hga_device_check: the check word could not be read");
    *word = w;
    return HGA_OK;
}

int hga_checked_build(void)
{
#ifdef HGA_CHECK_BOUNDS
    return 1;
#else
    return 0;
#endif
}

int hga_selftest_wait(int limit_us, int* site, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_selftest_wait");
    if (limit_us < 1 || limit_us > 1000000)
        return fail(HGA_ERR_INVALID_ARG, "limit_us=%d outside [1, 1000000]", limit_us);
    if (site) *site = hga::selftest_site();
    const cudaError_t e = hga::launch_selftest_wait(1000ull * (unsigned long long)limit_us,
                                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_selftest_wait");
}

int hga_route_widths(const hga_params* p, int* wc, int* wg)
{
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (!wc || !wg) return fail(HGA_ERR_INVALID_ARG, "wc / wg output pointer is NULL");
    *wc = s.wc;
    *wg = s.wg;
    return HGA_OK;
}

size_t hga_workspace_size(const hga_params* p)
{
    hga::Shape s{};
    if (make_shape(p, &s)) return 0;
    return sizeof(float) * (size_t)hga::bwd_scratch_floats(s);
}

int hga_build_summaries(const hga_params* p, const void* K, int64_t t_begin, int64_t t_end,
                        float* csum, float* gsum, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_build_summaries");
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (t_begin < 0 || t_end < t_begin || t_end > s.T || t_begin % 64 || t_end % 64)
        return fail(HGA_ERR_INVALID_ARG, "need 0 <= t_begin <= t_end <= T with multiples of 64 (got %lld, %lld, T=%lld)",
                    (long long)t_begin, (long long)t_end, (long long)s.T);
    if (t_end == t_begin) return HGA_OK;
    CHECK_PTR(K);
    CHECK_PTR(csum);
    CHECK_PTR(gsum);
    cudaError_t e = hga::launch_summaries(s, K, s.cap, 0, t_begin / 64, t_end / 64, csum, gsum,
                                          static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_build_summaries");
}

int hga_build_summaries_rows(const hga_params* p, const void* K_rows, int64_t t_begin, int64_t t_end,
                             float* csum, float* gsum, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_build_summaries_rows");
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (t_begin < 0 || t_end < t_begin || t_end > s.T || t_begin % 64 || t_end % 64)
        return fail(HGA_ERR_INVALID_ARG, "need 0 <= t_begin <= t_end <= T with multiples of 64 (got %lld, %lld, T=%lld)",
                    (long long)t_begin, (long long)t_end, (long long)s.T);
    if (t_end == t_begin) return HGA_OK;
    CHECK_PTR(K_rows);
    CHECK_PTR(csum);
    CHECK_PTR(gsum);
    cudaError_t e = hga::launch_summaries(s, K_rows, t_end - t_begin, t_begin, t_begin / 64, t_end / 64, csum,
                                          gsum, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_build_summaries_rows");
}

int hga_route_chunks(const hga_params* p, const void* Q, const float* csum, float* qbar,
                     int32_t* cidx, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_route_chunks");
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (s.nQB == 0) return HGA_OK;
    CHECK_PTR(Q);
    CHECK_PTR(csum);
    CHECK_PTR(qbar);
    CHECK_PTR(cidx);
    if (hga::route_chunks_smem(s) > kMaxSmem)
        return fail(HGA_ERR_UNSUPPORTED, "context of %lld chunks exceeds the chunk router's shared memory",
                    (long long)s.nC);
    cudaError_t e = hga::launch_route_chunks(s, Q, csum, qbar, cidx, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_route_chunks");
}

int hga_route_groups(const hga_params* p, const float* qbar, const float* gsum, const int32_t* cidx,
                     int32_t* gidx, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_route_groups");
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (s.nQB == 0) return HGA_OK;
    CHECK_PTR(qbar);
    CHECK_PTR(gsum);
    CHECK_PTR(cidx);
    CHECK_PTR(gidx);
    if (hga::route_groups_smem(s) > kMaxSmem)
        return fail(HGA_ERR_UNSUPPORTED, "k_c=%d gives too many candidate groups for the group router", s.wc);
    cudaError_t e = hga::launch_route_groups(s, qbar, gsum, cidx, gidx, static_cast<cudaStream_t>(stream));
    return finish(e, static_cast<cudaStream_t>(stream), "hga_route_groups");
}

int hga_route(const hga_params* p, const void* Q, const float* csum, const float* gsum, float* qbar,
              int32_t* cidx, int32_t* gidx, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_route");
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (s.nQB == 0) return HGA_OK;
    CHECK_PTR(Q);
    CHECK_PTR(csum);
    CHECK_PTR(gsum);
    CHECK_PTR(qbar);
    CHECK_PTR(cidx);
    CHECK_PTR(gidx);
    if (hga::route_fused_smem(s) > kMaxSmem)
        return fail(HGA_ERR_UNSUPPORTED, "routing of %lld chunks / k_c=%d exceeds the router's shared memory",
                    (long long)s.nC, s.wc);
    cudaError_t e = hga::launch_route_fused(s, Q, csum, gsum, qbar, cidx, gidx, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_route");
}

int hga_stage_params(const hga_params* p, hga_params* staged)
{
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (!staged) return fail(HGA_ERR_INVALID_ARG, "staged is NULL");
    *staged = *p;
    staged->T_hist = hga::stage_hist_rows(s);
    staged->kv_capacity = 0;                   // the staging buffers are dense
    // The staged problem keeps the routing's row widths: with HGA_ALL they
    // would otherwise follow the staged T.
    staged->k_c = s.wc;
    staged->k_g = s.wg;
    return HGA_OK;
}

int hga_stage_routed(const hga_params* p, const void* K_hist, const void* V_hist, const void* K_seg,
                     const void* V_seg, const int32_t* gidx, void* K_stage, void* V_stage, int32_t* gidx_stage,
                     hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_stage_routed");
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (s.nQB == 0) return HGA_OK;
    if (s.T_hist > 0) {
        CHECK_PTR(K_hist);
        CHECK_PTR(V_hist);
    }
    CHECK_PTR(K_seg);
    CHECK_PTR(V_seg);
    CHECK_PTR(gidx);
    CHECK_PTR(K_stage);
    CHECK_PTR(V_stage);
    CHECK_PTR(gidx_stage);
    const void* kh = K_hist;
    const void* vh = V_hist;
    if (s.T_hist > 0) {
        if (int r = device_addressable(K_hist, &kh, "K_hist")) return r;
        if (int r = device_addressable(V_hist, &vh, "V_hist")) return r;
    }
    const cudaError_t e = hga::launch_stage(s, kh, vh, K_seg, V_seg, gidx, K_stage, V_stage, gidx_stage,
                                            static_cast<cudaStream_t>(stream));
    return finish(e, static_cast<cudaStream_t>(stream), "hga_stage_routed");
}

int hga_decode(const hga_params* p, int64_t pos, const void* q, const void* K, const void* V,
               const float* csum, const float* gsum, float* O, float* lse, int32_t* cidx, int32_t* gidx,
               hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_decode");
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (pos < 0 || pos >= s.T)
        return fail(HGA_ERR_INVALID_ARG, "pos (%lld) must lie in [0, T=%lld)", (long long)pos, (long long)s.T);
    CHECK_PTR(q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(csum);
    CHECK_PTR(gsum);
    CHECK_PTR(O);
    CHECK_PTR(lse);
    CHECK_PTR(cidx);
    CHECK_PTR(gidx);
    if (s.G > hga::decode_max_heads())
        return fail(HGA_ERR_UNSUPPORTED, "decode takes at most %d q-heads per kv-head (got %d)",
                    hga::decode_max_heads(), s.G);
    if (hga::decode_smem(s) + 1024 > kMaxSmem)      // + the kernel's static shared memory
        return fail(HGA_ERR_UNSUPPORTED, "decode of %lld chunks / k_g=%d exceeds the kernel's shared memory",
                    (long long)s.nC, s.wg);
    cudaError_t e = hga::launch_decode(s, pos, q, K, V, csum, gsum, O, lse, cidx, gidx,
                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_decode");
}

// Shared checks of the causal variant's calls.
static int causal_shape(const hga_params* p, hga::Shape* s)
{
    if (int r = make_shape(p, s)) return r;
    if (s->G > hga::causal_max_heads())
        return fail(HGA_ERR_UNSUPPORTED, "the causal variant takes at most %d q-heads per kv-head (got %d)",
                    hga::causal_max_heads(), s->G);
    return HGA_OK;
}

int hga_route_causal(const hga_params* p, const void* Q, const float* csum, const float* gsum, int32_t* cidx,
                     int32_t* gidx, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_route_causal");
    hga::Shape s{};
    if (int r = causal_shape(p, &s)) return r;
    if (s.nQB == 0) return HGA_OK;
    CHECK_PTR(Q);
    CHECK_PTR(csum);
    CHECK_PTR(gsum);
    CHECK_PTR(cidx);
    CHECK_PTR(gidx);
    if (hga::route_causal_smem(s) + 1024 > kMaxSmem)
        return fail(HGA_ERR_UNSUPPORTED, "causal routing of %lld chunks / k_c=%d exceeds shared memory",
                    (long long)s.nC, s.wc);
    cudaError_t e = hga::launch_route_causal(s, Q, csum, gsum, cidx, gidx, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_route_causal");
}

size_t hga_causal_sched_size(const hga_params* p)
{
    hga::Shape s{};
    if (causal_shape(p, &s)) return 0;
    return 2 * sizeof(int32_t) * (size_t)hga::causal_items(s);
}

int hga_causal_schedule(const hga_params* p, const int32_t* gidx, int32_t* sched, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_causal_schedule");
    hga::Shape s{};
    if (int r = causal_shape(p, &s)) return r;
    if (hga::causal_items(s) == 0) return HGA_OK;
    CHECK_PTR(gidx);
    CHECK_PTR(sched);
    if (hga::causal_items(s) > INT32_MAX / 2)
        return fail(HGA_ERR_UNSUPPORTED, "%lld window items exceed the schedule's int32 range",
                    (long long)hga::causal_items(s));
    if (hga::causal_sched_smem(s) + 1024 > kMaxSmem)
        return fail(HGA_ERR_UNSUPPORTED, "the schedule's bitmap of %lld groups exceeds shared memory",
                    (long long)s.nG);
    cudaError_t e = hga::launch_causal_schedule(s, gidx, sched, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_causal_schedule");
}

int hga_attn_fwd_causal(const hga_params* p, const void* Q, const void* K, const void* V, const int32_t* gidx,
                        const int32_t* sched, float* O, float* lse, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_attn_fwd_causal");
    hga::Shape s{};
    if (int r = causal_shape(p, &s)) return r;
    if (s.nQB == 0) return HGA_OK;
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(gidx);
    if (sched) CHECK_PTR(sched);
    CHECK_PTR(O);
    CHECK_PTR(lse);
    cudaError_t e = hga::launch_attn_fwd_causal(s, Q, K, V, gidx, sched, O, lse, static_cast<cudaStream_t>(stream));
    return finish(e, static_cast<cudaStream_t>(stream), "hga_attn_fwd_causal");
}

int hga_attn_bwd_causal(const hga_params* p, const void* Q, const void* K, const void* V, const float* O,
                        const float* lse, const void* dO, const int32_t* gidx, const int32_t* sched, float* dQ,
                        float* dK_seg, float* dV_seg, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_attn_bwd_causal");
    hga::Shape s{};
    if (int r = causal_shape(p, &s)) return r;
    if (s.nQB == 0) return HGA_OK;
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(O);
    CHECK_PTR(lse);
    CHECK_PTR(dO);
    CHECK_PTR(gidx);
    if (sched) CHECK_PTR(sched);
    CHECK_PTR(dQ);
    CHECK_PTR(dK_seg);
    CHECK_PTR(dV_seg);
    cudaError_t e = hga::launch_attn_bwd_causal(s, Q, K, V, O, lse, dO, gidx, sched, dQ, dK_seg, dV_seg,
                                                static_cast<cudaStream_t>(stream));
    return finish(e, static_cast<cudaStream_t>(stream), "hga_attn_bwd_causal");
}

int hga_attn_fwd(const hga_params* p, const void* Q, const void* K, const void* V,
                 const int32_t* gidx, float* O, float* lse, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_attn_fwd");
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (s.nQB == 0) return HGA_OK;
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(gidx);
    CHECK_PTR(O);
    CHECK_PTR(lse);
    if (!hga::attn_fwd_tc_supported(s) && hga::attn_simt_smem(s, false) > kMaxSmem)
        return fail(HGA_ERR_UNSUPPORTED, "k_g=%d too large for the attention kernel", s.wg);
    // bf16: tcgen05 tensor-core kernel; float32: the FMA kernel (1e-4 gate).
    cudaError_t e = hga::attn_fwd_tc_supported(s)
                        ? hga::launch_attn_fwd_tc(s, Q, K, V, gidx, O, lse, static_cast<cudaStream_t>(stream))
                        : hga::launch_attn_fwd_simt(s, Q, K, V, gidx, O, lse, static_cast<cudaStream_t>(stream));
    return finish(e, static_cast<cudaStream_t>(stream), "hga_attn_fwd");
}

int hga_route_attn_fwd(const hga_params* p, const void* Q, const void* K, const void* V, const float* csum,
                       const float* gsum, float* qbar, int32_t* cidx, int32_t* gidx, float* O, float* lse,
                       hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_route_attn_fwd");
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (s.nQB == 0) return HGA_OK;
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(csum);
    CHECK_PTR(gsum);
    CHECK_PTR(qbar);
    CHECK_PTR(cidx);
    CHECK_PTR(gidx);
    CHECK_PTR(O);
    CHECK_PTR(lse);
    const auto st = static_cast<cudaStream_t>(stream);
    if (hga::route_attn_fwd_tc_supported(s))
        return finish(hga::launch_route_attn_fwd_tc(s, Q, K, V, csum, gsum, qbar, cidx, gidx, O, lse, st), st,
                      "hga_route_attn_fwd");
    // Other shapes: the router's launch, then the forward's (the same results).
    if (hga::route_fused_smem(s) > kMaxSmem)
        return fail(HGA_ERR_UNSUPPORTED, "routing of %lld chunks / k_c=%d exceeds the router's shared memory",
                    (long long)s.nC, s.wc);
    if (!hga::attn_fwd_tc_supported(s) && hga::attn_simt_smem(s, false) > kMaxSmem)
        return fail(HGA_ERR_UNSUPPORTED, "k_g=%d too large for the attention kernel", s.wg);
    cudaError_t e = hga::launch_route_fused(s, Q, csum, gsum, qbar, cidx, gidx, st);
    if (e == cudaSuccess)
        e = hga::attn_fwd_tc_supported(s) ? hga::launch_attn_fwd_tc(s, Q, K, V, gidx, O, lse, st)
                                          : hga::launch_attn_fwd_simt(s, Q, K, V, gidx, O, lse, st);
    return finish(e, st, "hga_route_attn_fwd");
}

int hga_attn_bwd(const hga_params* p, const void* Q, const void* K, const void* V, const float* O,
                 const float* lse, const void* dO, const int32_t* gidx, float* dQ, float* dK_seg,
                 float* dV_seg, void* workspace, size_t ws_bytes, hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_attn_bwd");
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (s.nQB == 0) return HGA_OK;
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(O);
    CHECK_PTR(lse);
    CHECK_PTR(dO);
    CHECK_PTR(gidx);
    CHECK_PTR(dQ);
    CHECK_PTR(dK_seg);
    CHECK_PTR(dV_seg);
    CHECK_PTR(workspace);
    const size_t need = sizeof(float) * (size_t)hga::bwd_scratch_floats(s);
    if (ws_bytes < need)
        return fail(HGA_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, need);
    if (!hga::attn_bwd_tc_supported(s) && hga::attn_simt_smem(s, true) > kMaxSmem)
        return fail(HGA_ERR_UNSUPPORTED, "k_g=%d too large for the attention kernel", s.wg);
    cudaError_t e = run_attn_bwd(s, Q, K, V, O, lse, dO, gidx, dQ, dK_seg, dV_seg, static_cast<float*>(workspace),
                                 static_cast<cudaStream_t>(stream));
    return finish(e, static_cast<cudaStream_t>(stream), "hga_attn_bwd");
}

}  // extern "C"

// ---- hga_attn_bwd_noalloc: the backward with built-in scratch -----------------
//
// Some callers cannot give this library a scratch buffer: plugin interfaces
// that hand an operator only its inputs and outputs, hosts whose memory pool
// owns every byte of device memory, and latency-bound loops that must not
// call cudaMalloc / cudaFree (cudaFree waits for the whole device).  For
// them the backward's only scratch, the per-row sums D = rowsum(dO * O), lives
// in the fixed array below, which the CUDA runtime places in device memory
// when the library's code is loaded on a device and frees at process exit.
// Host code must not use the array's name as a pointer: on the host it is a
// stand-in symbol, not a device address.  Its device address is looked up
// once per device with cudaGetSymbolAddress, on the first call made while
// that device is current, and cached.

// Size of the built-in scratch in 4-byte words: the row sums of up to
// HGA_NOALLOC_MAX_ROWS rows, then the backward's item schedule.  An item is
// a query block of 64 rows of at least one q-head, so the schedule holds at
// most one word per 64 rows; the call below checks the exact need,
// hga::bwd_scratch_floats, against this total, so a change in how items are
// counted cannot overrun the array.
constexpr int64_t kNoallocWords = (int64_t)HGA_NOALLOC_MAX_ROWS + HGA_NOALLOC_MAX_ROWS / 64;
static __device__ __align__(256) float g_noalloc_rowsum[kNoallocWords];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_rowsum on the current device (looked up once).
int noalloc_scratch(float** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "hga_attn_bwd_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices)
        return fail(HGA_ERR_UNSUPPORTED, "hga_attn_bwd_noalloc: device %d beyond the %d supported", dev,
                    kMaxDevices);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
        void* addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_noalloc_rowsum);
        if (e != cudaSuccess) return cuda_fail(e, "hga_attn_bwd_noalloc: cudaGetSymbolAddress");
        g_noalloc_addr[dev] = static_cast<float*>(addr);
    }
    *out = g_noalloc_addr[dev];
    return HGA_OK;
}

}  // namespace

extern "C" int hga_attn_bwd_noalloc(const hga_params* p, const void* Q, const void* K, const void* V,
                                    const float* O, const float* lse, const void* dO,
                                    const int32_t* gidx, float* dQ, float* dK_seg, float* dV_seg,
                                    hga_stream_t stream)
{
    const NvtxRange nvtx_range("hga_attn_bwd_noalloc");
    hga::Shape s{};
    if (int r = make_shape(p, &s)) return r;
    if (s.nQB == 0) return HGA_OK;
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(O);
    CHECK_PTR(lse);
    CHECK_PTR(dO);
    CHECK_PTR(gidx);
    CHECK_PTR(dQ);
    CHECK_PTR(dK_seg);
    CHECK_PTR(dV_seg);
    const int64_t rows = (int64_t)s.B * s.Hq * s.T_seg;
    if (rows > HGA_NOALLOC_MAX_ROWS || hga::bwd_scratch_floats(s) > kNoallocWords)
        return fail(HGA_ERR_INVALID_ARG,
                    "hga_attn_bwd_noalloc: B*Hq*T_seg = %lld (%lld scratch words) exceeds its built-in "
                    "scratch of %d rows (%lld words); use hga_attn_bwd with a caller-provided workspace",
                    (long long)rows, (long long)hga::bwd_scratch_floats(s), HGA_NOALLOC_MAX_ROWS,
                    (long long)kNoallocWords);
    if (!hga::attn_bwd_tc_supported(s) && hga::attn_simt_smem(s, true) > kMaxSmem)
        return fail(HGA_ERR_UNSUPPORTED, "k_g=%d too large for the attention kernel", s.wg);
    float* scratch = nullptr;
    if (int r = noalloc_scratch(&scratch)) return r;
    // Every row sum the kernels read is first written by this call, so the
    // scratch needs no clearing between calls.
    cudaError_t e = run_attn_bwd(s, Q, K, V, O, lse, dO, gidx, dQ, dK_seg, dV_seg, scratch,
                                 static_cast<cudaStream_t>(stream));
    return finish(e, static_cast<cudaStream_t>(stream), "hga_attn_bwd_noalloc");
}
