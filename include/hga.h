/*
 * hga.h -- C ABI of libhga.so: Hierarchical Global Attention (HGA), the
 * two-level routed sparse attention, on NVIDIA B200 (sm_100a).
 *
 * Method source: the article "BMW's 16 GB GPU just did what needs an A100"
 * (seventnews.com), section "What HGA does differently": the context is cut
 * into 64-token chunks whose compact summary vectors stay in device memory;
 * each query block scores the chunk summaries and keeps the top-k chunks,
 * opens them at the level of 8-token groups and keeps the top-k groups, and
 * attends the exact token K/V of the selected groups only.  Summaries steer
 * selection and are never attended to; the router has no learned weights.
 * The segment-wise backward of the same section detaches older KV: later
 * segments attend earlier exact tokens, but no gradient reaches them.
 *
 * Readings where the article is silent: a summary is the arithmetic mean of
 * the keys; a routing score is the plain dot product of the block query with
 * a summary; the block query is the mean of the block's 64 queries over every
 * q-head that shares the kv-head (GQA); routed chunks lie strictly before the
 * block's own chunk, which is always attended with the token-causal mask;
 * group routing is one top-k over all groups of the chosen chunks; equal
 * scores go to the lower index; fewer eligible candidates than k keep them
 * all and pad with -1.
 *
 * Conventions of every call
 *   - All tensors are dense row-major arrays in device memory of the current
 *     device, 16-byte aligned.  Shapes use: B batch, Hq q-heads, Hkv kv-heads
 *     (q-head h uses kv-head h / (Hq/Hkv)), d head dim, T_hist detached
 *     history length, T_seg active segment length, T = T_hist + T_seg,
 *     nQB = T_seg / 64 query blocks.
 *       Q, dO      [B][Hq][T_seg][d]    (dtype of hga_params.dtype)
 *       K, V       [B][Hkv][T][d]       (dtype; segment keys at [T_hist, T))
 *       csum       [B][Hkv][T/64][d]    float32 chunk summaries
 *       gsum       [B][Hkv][T/8][d]     float32 group summaries
 *       qbar       [B][Hkv][nQB][d]     float32 block queries
 *       cidx       [B][Hkv][nQB][wc]    int32 chosen chunks (hga_route_widths)
 *       gidx       [B][Hkv][nQB][wg]    int32 chosen groups
 *       O          [B][Hq][T_seg][d]    float32
 *       lse        [B][Hq][T_seg]       float32, natural log of sum exp
 *       dQ         [B][Hq][T_seg][d]    float32
 *       dK_seg, dV_seg [B][Hkv][T_seg][d] float32 (segment keys only)
 *     Index rows hold global chunk / group numbers within their (b, kv-head),
 *     ascending, then -1 padding.
 *   - The caller owns all memory.  The library allocates nothing, never
 *     synchronises, and enqueues its kernels on `stream` (a cudaStream_t;
 *     NULL is the legacy default stream).  Calls return before the work is
 *     done.
 *   - Return value: HGA_OK, or an error code.  Arguments are validated on the
 *     host before any launch; on error nothing is launched and
 *     hga_last_error() gives a message (per calling thread).
 */
#ifndef HGA_H
#define HGA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HGA_OK               0
#define HGA_ERR_INVALID_ARG  1  /* bad shape, pointer, alignment or range   */
#define HGA_ERR_UNSUPPORTED  2  /* valid but not implemented (e.g. d = 96)  */
#define HGA_ERR_CUDA         3  /* a launch failed (message has the detail) */
#define HGA_ERR_DEVICE_CHECK 4  /* checked build: a device bounds check failed */

#define HGA_ALL  (-1)           /* k_c / k_g: keep every eligible candidate */

#define HGA_BF16 0              /* Q, K, V, dO are bfloat16                  */
#define HGA_FP32 1              /* Q, K, V, dO are float32                   */

typedef void* hga_stream_t;     /* a cudaStream_t                            */

typedef struct hga_params {
    int     B, Hq, Hkv, d;      /* d in {64, 128}; Hq % Hkv == 0             */
    int64_t T_hist, T_seg;      /* multiples of 64; T_seg may be 0 (no work) */
    int     chunk, group, qblock; /* must be 64, 8, 64                        */
    int     k_c, k_g;           /* >= 1, or HGA_ALL                          */
    float   scale;              /* softmax scale; 0 selects 1/sqrt(d)        */
    int     dtype;              /* HGA_BF16 or HGA_FP32                      */
    int64_t kv_capacity;        /* rows per (batch, kv-head) of the K / V
                                 * buffers; 0 = T_hist + T_seg (see below)   */
} hga_params;

/* kv_capacity lets a caller keep K / V in a preallocated cache that grows
 * segment by segment: K and V are [B][Hkv][kv_capacity][d] with rows
 * 0 .. T_hist + T_seg - 1 of each (batch, kv-head) in use, and the chunk /
 * group summaries are [B][Hkv][kv_capacity / 64][d] and
 * [B][Hkv][kv_capacity / 8][d].  It must be 0 or a multiple of 64 that is
 * at least T_hist + T_seg.  It applies to every K, V, csum and gsum
 * argument below, except K_rows of hga_build_summaries_rows (its own rows)
 * and the history / segment rows that hga_stage_routed reads (dense). */

/* Row widths of the index tables: wc = k_c (T/64 for HGA_ALL); wg = k_g
 * (8 * wc for HGA_ALL).  Returns HGA_OK or HGA_ERR_INVALID_ARG. */
int hga_route_widths(const hga_params* p, int* wc, int* wg);

/* Bytes of device scratch that hga_attn_bwd needs: B*Hq*T_seg floats for
 * the per-row sums D = rowsum(dO * O), then one int32 per work item of the
 * backward (B*Hkv*(T_seg/64)*ceil(G/2), G = Hq/Hkv) for its schedule.  0 on
 * invalid parameters. */
size_t hga_workspace_size(const hga_params* p);

/* a1. Chunk and group summaries: the mean of each 64-token chunk and of each
 * 8-token group of K (article section "What HGA does differently": compact
 * summary vectors of each chunk stay in device memory).  Only tokens
 * [t_begin, t_end) are summarised (multiples of 64, 0 <= t_begin <= t_end
 * <= T); the other rows of csum / gsum are left untouched, so a segment
 * step appends the summaries of its own keys to those kept from earlier
 * segments.  Accumulates in float32. */
int hga_build_summaries(const hga_params* p, const void* K, int64_t t_begin,
                        int64_t t_end, float* csum, float* gsum,
                        hga_stream_t stream);

/* a1 for callers that hold only the rows being summarised on the device
 * (e.g. with the history in host memory, see hga_stage_routed): the same as
 * hga_build_summaries, but K_rows is [B][Hkv][t_end - t_begin][d] and holds
 * tokens t_begin .. t_end-1 only. */
int hga_build_summaries_rows(const hga_params* p, const void* K_rows,
                             int64_t t_begin, int64_t t_end, float* csum,
                             float* gsum, hga_stream_t stream);

/* a2 + a3. Block queries and chunk routing (same section: the query scores
 * the chunk summaries and picks the top-k chunks).  Writes qbar (the mean
 * of the block's queries over the G q-heads of each kv-head) and cidx: for
 * block qb with own chunk c0 = T_hist/64 + qb, the min(k_c, c0) chunks
 * c < c0 of highest score qbar . csum[c] (float32), ties to the lower index,
 * ascending, -1 padded to wc. */
int hga_route_chunks(const hga_params* p, const void* Q, const float* csum,
                     float* qbar, int32_t* cidx, hga_stream_t stream);

/* a4. Group routing (same section: it opens those chunks at the level of
 * 8-token groups).  Candidates are the 8 groups of every chunk in the cidx
 * row; keeps the k_g of highest score qbar . gsum[j] (float32), ties to
 * the lower index, ascending, -1 padded to wg. */
int hga_route_groups(const hga_params* p, const float* qbar, const float* gsum,
                     const int32_t* cidx, int32_t* gidx, hga_stream_t stream);

/* a2 + a3 + a4 in one launch: the same qbar, cidx and gidx as
 * hga_route_chunks followed by hga_route_groups (bit for bit), without the
 * round trip of qbar and cidx through device memory between the stages. */
int hga_route(const hga_params* p, const void* Q, const float* csum,
              const float* gsum, float* qbar, int32_t* cidx, int32_t* gidx,
              hga_stream_t stream);

/* a5. Routed attention forward (same section: only the exact token K/V of
 * the selected groups is loaded for the attention).  Query i of block qb
 * (global position p = T_hist + 64 qb + i) of q-head h attends the 8 tokens
 * of every group in gidx[b][h/G][qb] plus tokens 64*(p/64) .. p of its own
 * chunk: O = softmax(scale * q K^T) V and lse = log sum exp(scale * q K^T).
 * bf16 inputs run on the tcgen05 tensor cores, float32 inputs on the CUDA
 * cores; accumulation and softmax are in float32 either way. */
int hga_attn_fwd(const hga_params* p, const void* Q, const void* K,
                 const void* V, const int32_t* gidx, float* O, float* lse,
                 hga_stream_t stream);

/* a2-a5 in one launch: the fused segment step's routing and forward
 * (article section "What HGA does differently": HGA as a drop-in attention
 * module run segment by segment).  Same arguments and results as
 * hga_route(p, Q, csum, gsum, qbar, cidx, gidx) followed by
 * hga_attn_fwd(p, Q, K, V, gidx, O, lse): qbar, cidx and gidx are written as
 * hga_route writes them, O and lse as hga_attn_fwd does, bit for bit.  For
 * bf16 inputs one persistent kernel runs both: each CTA takes query
 * blocks, routes one (warps 0-7 run the router's steps) and runs the
 * forward of the block's q-head pairs on the routing it keeps in shared
 * memory.  Other shapes run the two launches.  Errors as hga_route and
 * hga_attn_fwd. */
int hga_route_attn_fwd(const hga_params* p, const void* Q, const void* K,
                       const void* V, const float* csum, const float* gsum,
                       float* qbar, int32_t* cidx, int32_t* gidx, float* O,
                       float* lse, hga_stream_t stream);

/* a6. Routed attention backward with the routing of the forward frozen
 * (same section: the router has no learned weights, so gradients reach the
 * projections as in the dense case; older KV is detached).  Given O and lse
 * of hga_attn_fwd and the upstream dO, writes dQ, and dK_seg / dV_seg for
 * the segment keys T_hist .. T-1 (overwritten, not accumulated), summed over
 * the G q-heads of each kv-head.  History keys receive no gradient.
 * `workspace` must hold hga_workspace_size(p) bytes of device memory. */
int hga_attn_bwd(const hga_params* p, const void* Q, const void* K,
                 const void* V, const float* O, const float* lse,
                 const void* dO, const int32_t* gidx, float* dQ,
                 float* dK_seg, float* dV_seg, void* workspace,
                 size_t ws_bytes, hga_stream_t stream);

/* Largest B*Hq*T_seg that hga_attn_bwd_noalloc accepts. */
#define HGA_NOALLOC_MAX_ROWS 1048576

/* hga_attn_bwd without the workspace argument.  The article has no
 * counterpart: this entry point exists for callers that cannot hand the
 * library any scratch memory -- plugin interfaces that pass an operator only
 * its inputs and outputs, hosts whose memory pool owns all device memory,
 * and loops that must not call cudaMalloc / cudaFree.  It computes what
 * hga_attn_bwd computes and allocates nothing: its scratch (B*Hq*T_seg
 * floats of row sums, then the backward's item schedule) is a fixed array
 * of HGA_NOALLOC_MAX_ROWS * 65 / 64 words (about 4 MiB) inside the library,
 * held on every device that loads the library until the process exits.
 *   - B*Hq*T_seg above HGA_NOALLOC_MAX_ROWS returns HGA_ERR_INVALID_ARG,
 *     with nothing launched.
 *   - The first call on a device (the calling thread's current device, which
 *     must own every pointer and the stream) looks up the array's device
 *     address with cudaGetSymbolAddress and caches it; make that first call
 *     before any stream capture on that device.
 *   - All calls on a device share the one array and every call overwrites
 *     the entries it uses before reading them.  Calls whose kernels overlap
 *     on the GPU (other streams, other threads) race on it: order them, e.g.
 *     on one stream. */
int hga_attn_bwd_noalloc(const hga_params* p, const void* Q, const void* K,
                         const void* V, const float* O, const float* lse,
                         const void* dO, const int32_t* gidx, float* dQ,
                         float* dK_seg, float* dV_seg, hga_stream_t stream);

/* Host-RAM KV tier (article section "How it fits in 16 GB": older KV can be
 * held in host RAM; after routing only the selected groups' exact tokens are
 * brought to the GPU).  The history rows of K and V (positions < T_hist)
 * may live in pinned host memory that the device can address (memory from
 * cudaHostAlloc / cudaMallocHost, or registered with cudaHostRegister with
 * the mapped flag) or in device memory; the segment rows, the summaries and
 * the index rows live in device memory as usual.
 *
 * hga_stage_params: the parameter block of the staged problem -- *staged =
 * *p with T_hist replaced by T_stage = round_up_64(nQB * wg * 8), the
 * number of staged history rows per (batch, kv-head), and k_c, k_g replaced
 * by the row widths wc, wg of p (hga_route_widths), so that the staged index
 * rows keep their width also under HGA_ALL. */
int hga_stage_params(const hga_params* p, hga_params* staged);

/* Gather, after routing, every routed history group into a device staging
 * buffer and rewrite the index rows, so that hga_attn_fwd / hga_attn_bwd
 * with the staged parameter block (hga_stage_params), K_stage, V_stage and
 * gidx_stage compute exactly what they compute on the full K, V and gidx.
 *   K_hist, V_hist  [B][Hkv][T_hist][d]  history rows (host-mapped or device)
 *   K_seg, V_seg    [B][Hkv][T_seg][d]   segment rows (device)
 *   gidx            [B][Hkv][nQB][wg]    routing of hga_route (device)
 *   K_stage, V_stage [B][Hkv][T_stage + T_seg][d] (device, written): the
 *       distinct history groups routed by any query block of the (batch,
 *       kv-head), each copied once, in ascending group order: the k-th of
 *       them at rows 8k .. 8k+7; the segment rows follow at T_stage.  Rows
 *       past the last distinct group are left untouched and never read.
 *   gidx_stage      [B][Hkv][nQB][wg] (device, written): a history group
 *       becomes its rank k among the distinct routed history groups, a
 *       segment group j' becomes T_stage/8 + j' - T_hist/8, padding stays
 *       -1; rows stay ascending.
 * The segment keys keep their offsets past the (staged) history, so
 * dK_seg / dV_seg of the staged backward are those of the full problem.
 * Host-resident history is read over the host link with plain loads.
 * HGA_ERR_INVALID_ARG if K_hist / V_hist are neither device memory nor
 * device-addressable host memory. */
int hga_stage_routed(const hga_params* p, const void* K_hist, const void* V_hist,
                     const void* K_seg, const void* V_seg, const int32_t* gidx,
                     void* K_stage, void* V_stage, int32_t* gidx_stage,
                     hga_stream_t stream);

/* f3. One decode step (article section "Retrieval: no degradation in the
 * dense baseline": HGA can generate too).  The token at position pos is a
 * query block of one: its block query is the mean of its G q-heads' queries
 * (per kv-head); chunks c < pos / 64 are routed on csum (top k_c), their
 * groups on gsum (top k_g), and each q-head attends the routed groups' exact
 * tokens plus its own chunk's tokens 64 * (pos / 64) .. pos.  The shapes of
 * hga_params describe the cache: T = T_hist + T_seg rows of capacity.
 *   q          [B][Hq][d]          dtype, the new token's queries
 *   K, V       [B][Hkv][T][d]      dtype, rows 0 .. pos valid (pos included)
 *   csum, gsum as above; rows of chunks c < pos / 64 (groups of them) valid
 *              -- append a chunk's summaries with hga_build_summaries (or
 *              hga_build_summaries_rows) once its 64 tokens are in the cache
 *   O          [B][Hq][d]          float32
 *   lse        [B][Hq]             float32, natural log
 *   cidx       [B][Hkv][wc]        int32 (widths of hga_route_widths)
 *   gidx       [B][Hkv][wg]        int32
 * Rows outside 0 .. pos are never read.  HGA_ERR_INVALID_ARG if pos is not
 * in [0, T); HGA_ERR_UNSUPPORTED for more than 8 q-heads per kv-head or when
 * the routing state (8 bytes per chunk of T, about 70 bytes per unit of
 * wc) exceeds shared memory.  Runs as one 8-CTA cluster per (batch,
 * kv-head). */
int hga_decode(const hga_params* p, int64_t pos, const void* q, const void* K,
               const void* V, const float* csum, const float* gsum, float* O,
               float* lse, int32_t* cidx, int32_t* gidx, hga_stream_t stream);

/* f1. Strictly causal variant (article section "The one real caveat:
 * causal leakage": a block's routing depends on the scores of several query
 * positions, so an earlier token sees later tokens through it; the authors
 * mention a strictly causal variant).  Here every query position routes on
 * its own query, a query block of one as in hga_decode: its block query is
 * the mean of its G q-heads' queries; chunks c < (T_hist + i) / 64 are
 * routed (top k_c), then their groups (top k_g); each q-head attends the
 * routed groups' exact tokens and its own chunk up to itself.  The output
 * at segment position i depends on positions <= i only.  Routing rows are
 * per position:
 *   cidx [B][Hkv][T_seg][wc], gidx [B][Hkv][T_seg][wg]   int32
 * and the other tensors are as for the block calls.  hga_attn_bwd_causal
 * zeroes dK_seg / dV_seg itself (they are accumulated with atomics, so
 * their float32 sums are not bit-reproducible run to run).  At most 8
 * q-heads per kv-head (HGA_ERR_UNSUPPORTED otherwise).
 *
 * Schedule.  The bf16 attention calls run one CTA per window item (32
 * neighbouring positions of a (batch, kv-head) and four of its q-heads),
 * over the union of the window's routed groups; an item's time grows with
 * that union, which the routing decides.  hga_causal_schedule orders the
 * items by cost, heaviest first, from gidx:
 *   sched      int32 [2 * n_items], n_items = B * Hkv * ceil(T_seg / 32)
 *              * ceil(G / 4); hga_causal_sched_size gives its bytes (0 for
 *              invalid parameters).  sched[0 .. n_items) is the order (a
 *              permutation of the items), sched[n_items ..) their costs.
 * Passing it to hga_attn_fwd_causal / hga_attn_bwd_causal changes only the
 * order in which the items run, not their results (dQ, O and lse are the
 * same bit for bit; dK / dV up to the order of their atomic sums); NULL runs
 * the items in index order, and the float32 kernels ignore it.  It must be
 * built from the gidx the attention calls are given.  Caller-owned device
 * memory, 16-byte aligned. */
int hga_route_causal(const hga_params* p, const void* Q, const float* csum,
                     const float* gsum, int32_t* cidx, int32_t* gidx,
                     hga_stream_t stream);
size_t hga_causal_sched_size(const hga_params* p);
int hga_causal_schedule(const hga_params* p, const int32_t* gidx,
                        int32_t* sched, hga_stream_t stream);
int hga_attn_fwd_causal(const hga_params* p, const void* Q, const void* K,
                        const void* V, const int32_t* gidx,
                        const int32_t* sched, float* O, float* lse,
                        hga_stream_t stream);
int hga_attn_bwd_causal(const hga_params* p, const void* Q, const void* K,
                        const void* V, const float* O, const float* lse,
                        const void* dO, const int32_t* gidx,
                        const int32_t* sched, float* dQ, float* dK_seg,
                        float* dV_seg, hga_stream_t stream);

/* Status word of the kernels' bounded waits: every wait of a tensor-core
 * kernel or of the decode kernel on a barrier gives up after one second, records the code of the wait
 * in this word and lets the kernel return (its outputs are then invalid).
 * *status = 0 when no wait ran out; `clear` != 0 resets the word.
 * Synchronises with the device. */
int hga_device_status(int* status, int clear);

/* Bounds-check build.  A library compiled with -DHGA_CHECK_BOUNDS
 * (libhga_checked.so) checks, on the device, every routed group or chunk
 * index it reads from a caller's index row before using it as an address
 * (valid: 0 <= index < the row's own chunk, in chunks or groups); an index
 * outside records a site code in a device check word and is replaced by
 * index 0 of the same (batch, kv-head) (the strictly causal tensor-core
 * kernels, which merge the index rows of 32 neighbouring positions, drop
 * it instead), so no access leaves the tensors.
 * In that build hga_route_groups, hga_attn_fwd, hga_attn_bwd,
 * hga_attn_bwd_noalloc, hga_stage_routed, hga_attn_fwd_causal and
 * hga_attn_bwd_causal wait for their stream and return HGA_ERR_DEVICE_CHECK
 * (outputs invalid, word cleared) when a check failed.  Release builds skip
 * the checks and return without waiting.
 * hga_checked_build: 1 in a checked build, else 0.
 * hga_device_check: *word = the first failed check's site code (0: none);
 * `clear` != 0 resets it.  Synchronises with the device. */
int hga_checked_build(void);
int hga_device_check(int* word, int clear);

/* Failure-path self-test.  The article has no counterpart: this call lets a
 * caller (or a test) check that the library's bounded waits end cleanly.
 * It launches one CTA on `stream` that allocates tensor memory, waits on an
 * mbarrier nothing arrives at until `limit_us` microseconds pass, records
 * its code (written to *site when site is not NULL) in the status word that
 * hga_device_status reads, frees the tensor memory and returns.  The device
 * stays usable.  HGA_ERR_INVALID_ARG unless 1 <= limit_us <= 1000000. */
int hga_selftest_wait(int limit_us, int* site, hga_stream_t stream);

/* Message of the last failed call on this thread ("" if none). */
const char* hga_last_error(void);

/* Library version string. */
const char* hga_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HGA_H */
