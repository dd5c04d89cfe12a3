/*
 * hga_oracle.c -- plain, slow, double-precision CPU oracle for Hierarchical
 * Global Attention (HGA) two-level routed sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA library; it is written from the method's definition, step by step,
 * with explicit loops, a full sort per routing row and no online softmax.
 *
 * Source of the method: the article "BMW's 16 GB GPU just did what needs an
 * A100" (seventnews.com), section "What HGA does differently":
 *   - the context is cut into 64-token chunks whose compact summary vectors
 *     stay on the device;
 *   - each query block scores the chunk summaries and keeps the top-k chunks,
 *     then opens those chunks at the level of 8-token groups and keeps the
 *     top-k groups;
 *   - exact token K/V of the selected groups is attended; summaries only
 *     steer selection and are never attended to;
 *   - the router has no learned weights (it scores the projected keys), so
 *     gradients reach Q/K/V as for dense attention.
 * Same article, section "The one real caveat: causal leakage": routing of a
 * block depends on the scores of several query positions.
 * Same article, section "What HGA does differently" (segment-wise backward):
 * gradients do not cross segment boundaries; later segments still attend to
 * earlier exact tokens, which are detached.
 *
 * Readings where the article is silent (each one is listed with its reason
 * in the design notes of the repository):
 *   R1 summary   = arithmetic mean of the keys of the chunk / group;
 *   R2 score     = plain dot product  qbar . summary  (no scale: ranking only);
 *   R3 qbar      = mean of the block's queries over all q-heads that share
 *                  the kv-head (GQA), i.e. over G*chunk query rows;
 *   R4 eligible  = chunks strictly before the block's own chunk c0; the own
 *                  chunk is always attended with the token-causal mask;
 *   R5 groups    = one top-k over all groups of all chosen chunks;
 *   R6 fewer eligible than k: take all, pad with -1;
 *   R7 ties      = higher score first, equal scores -> lower index first;
 *                  the kept indices are reported in ascending order;
 *   R8 gap       = (s_k - s_{k+1}) / max(|s_k|, |s_{k+1}|, 1e-3*rms(scores))
 *                  of the (k)th and (k+1)th best scores, +inf if no (k+1)th;
 *   R9 softmax   = natural-log LSE, scale given by the caller (1/sqrt(d));
 *   R10 backward = routing frozen (non-differentiable); dK/dV summed over the
 *                  G q-heads of a kv-head and kept for segment keys only.
 *
 * Parity of this oracle against the authors' own implementation is not
 * pinnable (no code or worked example is published); it is pinned against
 * the definition by the CPU test-suite (brute force, closed forms, dense
 * equivalence, library attention and autograd, finite differences).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Problem description shared by every oracle entry point.  Layouts (row
 * major):  Q, dO, O, dQ  [B][Hq][T_seg][d];  K, V  [B][Hkv][T][d] with
 * T = T_hist + T_seg (segment keys at [T_hist, T));  csum [B][Hkv][T/chunk][d];
 * gsum [B][Hkv][T/group][d];  qbar [B][Hkv][T_seg/chunk][d];
 * cidx [B][Hkv][nQB][wc];  gidx [B][Hkv][nQB][wg];  lse [B][Hq][T_seg];
 * dK_seg, dV_seg [B][Hkv][T_seg][d]. */
typedef struct {
    int B, Hq, Hkv, d;
    int64_t T_hist, T_seg;
    int chunk, group;   /* query block == chunk */
    int k_c, k_g;       /* number to keep; <= 0 means "all eligible" */
    int wc, wg;         /* row widths of cidx / gidx (>= k_c, k_g) */
    double scale;
} oracle_dims;

static int64_t total_len(const oracle_dims* p) { return p->T_hist + p->T_seg; }

/* ---------------------------------------------------------------- a1 ---- */
/* Chunk and group summaries of the keys in [t_begin, t_end) (reading R1). */
void oracle_build_summaries(const oracle_dims* p, const double* K,
                            int64_t t_begin, int64_t t_end,
                            double* csum, double* gsum)
{
    const int64_t T = total_len(p);
    const int d = p->d;
    const int64_t nC = T / p->chunk, nG = T / p->group;
    for (int b = 0; b < p->B; ++b)
        for (int g = 0; g < p->Hkv; ++g) {
            const double* Kh = K + ((int64_t)b * p->Hkv + g) * T * d;
            double* cs = csum + ((int64_t)b * p->Hkv + g) * nC * d;
            double* gs = gsum + ((int64_t)b * p->Hkv + g) * nG * d;
            for (int64_t c = t_begin / p->chunk; c < t_end / p->chunk; ++c)
                for (int e = 0; e < d; ++e) {
                    double acc = 0.0;
                    for (int t = 0; t < p->chunk; ++t)
                        acc += Kh[(c * p->chunk + t) * d + e];
                    cs[c * d + e] = acc / p->chunk;
                }
            for (int64_t j = t_begin / p->group; j < t_end / p->group; ++j)
                for (int e = 0; e < d; ++e) {
                    double acc = 0.0;
                    for (int t = 0; t < p->group; ++t)
                        acc += Kh[(j * p->group + t) * d + e];
                    gs[j * d + e] = acc / p->group;
                }
        }
}

/* ---------------------------------------------------------------- a2 ---- */
/* Block query (reading R3): mean over the G q-heads of kv-head g and the
 * `chunk` queries of block qb. */
void oracle_block_query(const oracle_dims* p, const double* Q, double* qbar)
{
    const int G = p->Hq / p->Hkv, d = p->d;
    const int64_t nQB = p->T_seg / p->chunk;
    for (int b = 0; b < p->B; ++b)
        for (int g = 0; g < p->Hkv; ++g)
            for (int64_t qb = 0; qb < nQB; ++qb)
                for (int e = 0; e < d; ++e) {
                    double acc = 0.0;
                    for (int hh = 0; hh < G; ++hh) {
                        const int h = g * G + hh;
                        const double* Qh = Q + ((int64_t)b * p->Hq + h) * p->T_seg * d;
                        for (int i = 0; i < p->chunk; ++i)
                            acc += Qh[(qb * p->chunk + i) * d + e];
                    }
                    qbar[(((int64_t)b * p->Hkv + g) * nQB + qb) * d + e] =
                        acc / ((double)G * p->chunk);
                }
}

/* -------------------------------------------------------- top-k helper -- */
typedef struct { double s; int64_t idx; } cand;

/* Order of reading R7: higher score first, ties to the lower index. */
static int cand_order(const void* a, const void* b)
{
    const cand* x = (const cand*)a;
    const cand* y = (const cand*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->idx < y->idx) ? -1 : (x->idx > y->idx) ? 1 : 0;
}

static int idx_ascending(const void* a, const void* b)
{
    const int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* Keep the best min(k, n) of the n candidates (k <= 0: keep all), write them
 * ascending into out[0..w) padded with -1, and return the gap of reading R8. */
static double select_top(cand* cs, int64_t n, int k, int32_t* out, int w)
{
    qsort(cs, (size_t)n, sizeof(cand), cand_order);
    const int64_t keep = (k <= 0 || (int64_t)k > n) ? n : (int64_t)k;
    for (int i = 0; i < w; ++i) out[i] = -1;
    for (int64_t i = 0; i < keep && i < w; ++i) out[i] = (int32_t)cs[i].idx;
    qsort(out, (size_t)(keep < w ? keep : w), sizeof(int32_t), idx_ascending);
    if (keep >= n || keep == 0) return INFINITY;
    double ss = 0.0;
    for (int64_t i = 0; i < n; ++i) ss += cs[i].s * cs[i].s;
    const double tau = 1e-3 * sqrt(ss / (double)n);
    const double a = cs[keep - 1].s, b = cs[keep].s;
    double den = fabs(a);
    if (fabs(b) > den) den = fabs(b);
    if (tau > den) den = tau;
    return den > 0.0 ? (a - b) / den : 0.0;
}

static double dot(const double* x, const double* y, int d)
{
    double acc = 0.0;
    for (int e = 0; e < d; ++e) acc += x[e] * y[e];
    return acc;
}

/* ---------------------------------------------------------------- a3 ---- */
/* Chunk routing (readings R2, R4, R6, R7, R8).  gap: [B][Hkv][nQB]. */
void oracle_route_chunks(const oracle_dims* p, const double* qbar,
                         const double* csum, int32_t* cidx, double* gap)
{
    const int d = p->d;
    const int64_t nQB = p->T_seg / p->chunk, nC = total_len(p) / p->chunk;
    const int64_t units = (int64_t)p->B * p->Hkv * nQB;
#pragma omp parallel for schedule(dynamic)
    for (int64_t u = 0; u < units; ++u) {
        const int64_t bg = u / nQB, qb = u % nQB;
        const int64_t c0 = p->T_hist / p->chunk + qb;   /* own chunk */
        const double* q = qbar + u * d;
        const double* cs = csum + bg * nC * d;
        cand* list = (cand*)malloc(sizeof(cand) * (size_t)(c0 > 0 ? c0 : 1));
        for (int64_t c = 0; c < c0; ++c) {
            list[c].s = dot(q, cs + c * d, d);
            list[c].idx = c;
        }
        gap[u] = select_top(list, c0, p->k_c, cidx + u * p->wc, p->wc);
        free(list);
    }
}

/* ---------------------------------------------------------------- a4 ---- */
/* Group routing over all groups of the chosen chunks (R5 and the above). */
void oracle_route_groups(const oracle_dims* p, const double* qbar,
                         const double* gsum, const int32_t* cidx,
                         int32_t* gidx, double* gap)
{
    const int d = p->d, gpc = p->chunk / p->group;
    const int64_t nQB = p->T_seg / p->chunk, nG = total_len(p) / p->group;
    const int64_t units = (int64_t)p->B * p->Hkv * nQB;
#pragma omp parallel for schedule(dynamic)
    for (int64_t u = 0; u < units; ++u) {
        const int64_t bg = u / nQB;
        const double* q = qbar + u * d;
        const double* gs = gsum + bg * nG * d;
        cand* list = (cand*)malloc(sizeof(cand) * (size_t)(p->wc * gpc + 1));
        int64_t n = 0;
        for (int i = 0; i < p->wc; ++i) {
            const int32_t c = cidx[u * p->wc + i];
            if (c < 0) continue;
            for (int r = 0; r < gpc; ++r) {
                const int64_t j = (int64_t)c * gpc + r;
                list[n].s = dot(q, gs + j * d, d);
                list[n].idx = j;
                ++n;
            }
        }
        gap[u] = select_top(list, n, p->k_g, gidx + u * p->wg, p->wg);
        free(list);
    }
}

/* Key set of query position i (0-based inside the segment) of one block:
 * the tokens of every selected group, then the own chunk up to i itself.
 * Returns the number of keys written to keys[]. */
static int64_t key_set(const oracle_dims* p, const int32_t* grow, int64_t i,
                       int64_t* keys)
{
    int64_t n = 0;
    for (int r = 0; r < p->wg; ++r) {
        if (grow[r] < 0) continue;
        for (int t = 0; t < p->group; ++t) keys[n++] = (int64_t)grow[r] * p->group + t;
    }
    const int64_t pos = p->T_hist + i;                  /* global position */
    const int64_t start = (pos / p->chunk) * p->chunk;  /* own chunk start */
    for (int64_t t = start; t <= pos; ++t) keys[n++] = t;
    return n;
}

/* ---------------------------------------------------------------- a5 ---- */
/* Exact softmax attention over the routed key set (reading R9).  The softmax
 * is evaluated directly: scores, their maximum, exponentials, their sum. */
static void attn_fwd_rows(const oracle_dims* p, const double* Q, const double* K,
                          const double* V, const int32_t* gidx, int per_row, double* O,
                          double* lse)
{
    const int G = p->Hq / p->Hkv, d = p->d;
    const int64_t T = total_len(p);
    /* routing rows per (b, kv-head): one per block, or one per position */
    const int64_t nR = per_row ? p->T_seg : p->T_seg / p->chunk;
    const int64_t maxkeys = (int64_t)p->wg * p->group + p->chunk;
    const int64_t rows = (int64_t)p->B * p->Hq * p->T_seg;
#pragma omp parallel
    {
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)maxkeys);
        double* s = (double*)malloc(sizeof(double) * (size_t)maxkeys);
#pragma omp for schedule(dynamic, 64)
        for (int64_t r = 0; r < rows; ++r) {
            const int64_t i = r % p->T_seg, bh = r / p->T_seg;
            const int b = (int)(bh / p->Hq), h = (int)(bh % p->Hq), g = h / G;
            const int64_t qr = per_row ? i : i / p->chunk;
            const int32_t* grow = gidx + (((int64_t)b * p->Hkv + g) * nR + qr) * p->wg;
            const double* q = Q + r * d;
            const double* Kh = K + ((int64_t)b * p->Hkv + g) * T * d;
            const double* Vh = V + ((int64_t)b * p->Hkv + g) * T * d;
            const int64_t n = key_set(p, grow, i, keys);
            double m = -INFINITY;
            for (int64_t j = 0; j < n; ++j) {
                s[j] = p->scale * dot(q, Kh + keys[j] * d, d);
                if (s[j] > m) m = s[j];
            }
            double l = 0.0;
            for (int64_t j = 0; j < n; ++j) { s[j] = exp(s[j] - m); l += s[j]; }
            double* o = O + r * d;
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            for (int64_t j = 0; j < n; ++j) {
                const double w = s[j] / l;
                for (int e = 0; e < d; ++e) o[e] += w * Vh[keys[j] * d + e];
            }
            lse[r] = m + log(l);
        }
        free(keys);
        free(s);
    }
}

void oracle_attn_fwd(const oracle_dims* p, const double* Q, const double* K,
                     const double* V, const int32_t* gidx, double* O, double* lse)
{
    attn_fwd_rows(p, Q, K, V, gidx, 0, O, lse);
}

/* ---------------------------------------------------------------- a6 ---- */
/* Backward of a5 with the routing frozen (R10).  P is recomputed from the
 * inputs (not from a stored O or LSE) and the softmax Jacobian is applied
 * in its textbook form dS_j = P_j (dP_j - sum_k P_k dP_k).  Gradients of
 * keys before T_hist (detached history) are dropped. */
static void attn_bwd_rows(const oracle_dims* p, const double* Q, const double* K,
                          const double* V, const double* dO, const int32_t* gidx,
                          int per_row, double* dQ, double* dK_seg, double* dV_seg)
{
    const int G = p->Hq / p->Hkv, d = p->d;
    const int64_t T = total_len(p);
    const int64_t nR = per_row ? p->T_seg : p->T_seg / p->chunk;
    const int64_t maxkeys = (int64_t)p->wg * p->group + p->chunk;
    const int64_t units = (int64_t)p->B * p->Hkv;
    memset(dK_seg, 0, sizeof(double) * (size_t)(units * p->T_seg * d));
    memset(dV_seg, 0, sizeof(double) * (size_t)(units * p->T_seg * d));
    /* Each (b, kv-head) owns its dK/dV slice and its q-heads' dQ rows. */
#pragma omp parallel for schedule(dynamic)
    for (int64_t u = 0; u < units; ++u) {
        const int b = (int)(u / p->Hkv), g = (int)(u % p->Hkv);
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)maxkeys);
        double* P = (double*)malloc(sizeof(double) * (size_t)maxkeys);
        double* dP = (double*)malloc(sizeof(double) * (size_t)maxkeys);
        const double* Kh = K + u * T * d;
        const double* Vh = V + u * T * d;
        double* dK = dK_seg + u * p->T_seg * d;
        double* dV = dV_seg + u * p->T_seg * d;
        for (int hh = 0; hh < G; ++hh) {
            const int h = g * G + hh;
            for (int64_t i = 0; i < p->T_seg; ++i) {
                const int64_t r = ((int64_t)b * p->Hq + h) * p->T_seg + i;
                const int32_t* grow = gidx + (u * nR + (per_row ? i : i / p->chunk)) * p->wg;
                const double* q = Q + r * d;
                const double* dout = dO + r * d;
                const int64_t n = key_set(p, grow, i, keys);
                double m = -INFINITY;
                for (int64_t j = 0; j < n; ++j) {
                    P[j] = p->scale * dot(q, Kh + keys[j] * d, d);
                    if (P[j] > m) m = P[j];
                }
                double l = 0.0;
                for (int64_t j = 0; j < n; ++j) { P[j] = exp(P[j] - m); l += P[j]; }
                double pdp = 0.0;
                for (int64_t j = 0; j < n; ++j) {
                    P[j] /= l;
                    dP[j] = dot(dout, Vh + keys[j] * d, d);
                    pdp += P[j] * dP[j];
                }
                double* dq = dQ + r * d;
                for (int e = 0; e < d; ++e) dq[e] = 0.0;
                for (int64_t j = 0; j < n; ++j) {
                    const double ds = P[j] * (dP[j] - pdp);
                    const double* k = Kh + keys[j] * d;
                    for (int e = 0; e < d; ++e) dq[e] += p->scale * ds * k[e];
                    if (keys[j] >= p->T_hist) {
                        const int64_t t = keys[j] - p->T_hist;
                        for (int e = 0; e < d; ++e) {
                            dK[t * d + e] += p->scale * ds * q[e];
                            dV[t * d + e] += P[j] * dout[e];
                        }
                    }
                }
            }
        }
        free(keys);
        free(P);
        free(dP);
    }
}

void oracle_attn_bwd(const oracle_dims* p, const double* Q, const double* K,
                     const double* V, const double* dO, const int32_t* gidx,
                     double* dQ, double* dK_seg, double* dV_seg)
{
    attn_bwd_rows(p, Q, K, V, dO, gidx, 0, dQ, dK_seg, dV_seg);
}

/* Routing of one query block of a single position whose own chunk is c0:
 * qbar (d values) against the chunk summaries csu [nC][d] and the group
 * summaries gsu [nG][d] of one (b, kv-head).  Chunks c < c0 (R4), top-k_c
 * (R6, R7) into crow [wc]; groups of the chosen chunks, top-k_g (R5) into
 * grow [wg]; gaps (R8) into *cgap, *ggap.  list: scratch of at least
 * max(c0, 1) + wc * (chunk / group) + 1 candidates. */
static void route_single(const oracle_dims* p, const double* qbar, const double* csu,
                         const double* gsu, int64_t c0, cand* list, int32_t* crow,
                         int32_t* grow, double* cgap, double* ggap)
{
    const int d = p->d, gpc = p->chunk / p->group;
    for (int64_t c = 0; c < c0; ++c) {
        list[c].s = dot(qbar, csu + c * d, d);
        list[c].idx = c;
    }
    *cgap = select_top(list, c0, p->k_c, crow, p->wc);
    int64_t n = 0;
    for (int i = 0; i < p->wc; ++i) {
        const int32_t c = crow[i];
        if (c < 0) continue;
        for (int r = 0; r < gpc; ++r) {
            const int64_t j = (int64_t)c * gpc + r;
            list[n].s = dot(qbar, gsu + j * d, d);
            list[n].idx = j;
            ++n;
        }
    }
    *ggap = select_top(list, n, p->k_g, grow, p->wg);
}

/* ------------------------------------------------------------ decode ---- */
/* One generation step (article section "Retrieval: no degradation in the
 * dense baseline": HGA itself can also do generation): the new token at position pos
 * is a query block of one.  q [B][Hq][d]; K, V [B][Hkv][T][d] with rows
 * 0..pos valid (pos < T = T_hist + T_seg, the capacity); csum / gsum as for
 * the segment calls, rows of the complete chunks < pos/chunk used.
 *   qbar  = mean of the token's query over the G q-heads of the kv-head (R3
 *           with a block of one);
 *   chunks c < c0 = pos / chunk eligible (R4), top-k_c (R6, R7), gap (R8);
 *   groups of the chosen chunks, top-k_g (R5);
 *   O, lse: exact softmax over the routed groups' tokens and the own chunk's
 *           tokens c0*chunk .. pos (R9).
 * Outputs: O [B][Hq][d], lse [B][Hq], cidx [B][Hkv][wc], gidx [B][Hkv][wg],
 * cgap, ggap [B][Hkv]. */
void oracle_decode(const oracle_dims* p, int64_t pos, const double* q, const double* K,
                   const double* V, const double* csum, const double* gsum, double* O,
                   double* lse, int32_t* cidx, int32_t* gidx, double* cgap, double* ggap)
{
    const int G = p->Hq / p->Hkv, d = p->d, gpc = p->chunk / p->group;
    const int64_t T = total_len(p), nC = T / p->chunk, nG = T / p->group;
    const int64_t c0 = pos / p->chunk;
    const int64_t units = (int64_t)p->B * p->Hkv;
#pragma omp parallel for schedule(dynamic)
    for (int64_t u = 0; u < units; ++u) {
        const int64_t b = u / p->Hkv, g = u % p->Hkv;
        double* qbar = (double*)malloc(sizeof(double) * (size_t)d);
        for (int e = 0; e < d; ++e) {
            double a = 0.0;
            for (int h = 0; h < G; ++h) a += q[((b * p->Hq) + g * G + h) * d + e];
            qbar[e] = a / (double)G;
        }
        /* chunk and group routing */
        cand* list = (cand*)malloc(sizeof(cand) * (size_t)((c0 > 0 ? c0 : 1) + p->wc * gpc + 1));
        route_single(p, qbar, csum + u * nC * d, gsum + u * nG * d, c0, list, cidx + u * p->wc,
                     gidx + u * p->wg, &cgap[u], &ggap[u]);
        free(list);
        /* attention of each q-head of the kv-head */
        const int32_t* grow = gidx + u * p->wg;
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)(p->wg * p->group + p->chunk));
        double* s = (double*)malloc(sizeof(double) * (size_t)(p->wg * p->group + p->chunk));
        int64_t nk = 0;
        for (int r = 0; r < p->wg; ++r) {
            if (grow[r] < 0) continue;
            for (int t = 0; t < p->group; ++t) keys[nk++] = (int64_t)grow[r] * p->group + t;
        }
        for (int64_t t = c0 * p->chunk; t <= pos; ++t) keys[nk++] = t;
        const double* Kh = K + u * T * d;
        const double* Vh = V + u * T * d;
        for (int h = 0; h < G; ++h) {
            const int64_t row = b * p->Hq + g * G + h;
            const double* qh = q + row * d;
            double m = -INFINITY;
            for (int64_t j = 0; j < nk; ++j) {
                s[j] = p->scale * dot(qh, Kh + keys[j] * d, d);
                if (s[j] > m) m = s[j];
            }
            double l = 0.0;
            for (int64_t j = 0; j < nk; ++j) { s[j] = exp(s[j] - m); l += s[j]; }
            double* o = O + row * d;
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            for (int64_t j = 0; j < nk; ++j) {
                const double w = s[j] / l;
                for (int e = 0; e < d; ++e) o[e] += w * Vh[keys[j] * d + e];
            }
            lse[row] = m + log(l);
        }
        free(keys);
        free(s);
        free(qbar);
    }
}

/* ------------------------------------------------------------ causal ---- */
/* Strictly causal variant.  Article section "The one real caveat: causal
 * leakage": a block's routing depends on the scores of several query
 * positions, so through the routing an earlier token sees the queries of
 * later tokens of its block; the authors mention a strictly causal variant
 * in the works without describing it.  Reading R14: every query position
 * routes on its own query, a query block of one exactly as in the decode
 * step -- qbar_i = mean of Q[., i] over the G q-heads of the kv-head, chunks
 * c < (T_hist + i) / chunk eligible (R4), groups of the chosen chunks (R5),
 * attention over the routed groups' tokens and the own chunk up to i (R9).
 * Then the output at position i depends on positions <= i only.
 * Routing rows per position: cidx [B][Hkv][T_seg][wc], gidx [B][Hkv][T_seg][wg],
 * cgap, ggap [B][Hkv][T_seg]. */
void oracle_causal_route(const oracle_dims* p, const double* Q, const double* csum,
                         const double* gsum, int32_t* cidx, int32_t* gidx, double* cgap,
                         double* ggap)
{
    const int G = p->Hq / p->Hkv, d = p->d, gpc = p->chunk / p->group;
    const int64_t T = total_len(p), nC = T / p->chunk, nG = T / p->group;
    const int64_t rows = (int64_t)p->B * p->Hkv * p->T_seg;
#pragma omp parallel
    {
        double* qbar = (double*)malloc(sizeof(double) * (size_t)d);
        cand* list = (cand*)malloc(sizeof(cand) * (size_t)(nC + 1 + p->wc * gpc));
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            const int64_t u = r / p->T_seg, i = r % p->T_seg;
            const int64_t b = u / p->Hkv, g = u % p->Hkv;
            for (int e = 0; e < d; ++e) {
                double a = 0.0;
                for (int h = 0; h < G; ++h) a += Q[((b * p->Hq + g * G + h) * p->T_seg + i) * d + e];
                qbar[e] = a / (double)G;
            }
            const int64_t c0 = (p->T_hist + i) / p->chunk;
            route_single(p, qbar, csum + u * nC * d, gsum + u * nG * d, c0, list, cidx + r * p->wc,
                         gidx + r * p->wg, &cgap[r], &ggap[r]);
        }
        free(qbar);
        free(list);
    }
}

/* Attention forward / backward of the causal variant: as a5 / a6 with the
 * routing row of position i (gidx [B][Hkv][T_seg][wg]). */
void oracle_causal_attn_fwd(const oracle_dims* p, const double* Q, const double* K,
                            const double* V, const int32_t* gidx, double* O, double* lse)
{
    attn_fwd_rows(p, Q, K, V, gidx, 1, O, lse);
}

void oracle_causal_attn_bwd(const oracle_dims* p, const double* Q, const double* K,
                            const double* V, const double* dO, const int32_t* gidx,
                            double* dQ, double* dK_seg, double* dV_seg)
{
    attn_bwd_rows(p, Q, K, V, dO, gidx, 1, dQ, dK_seg, dV_seg);
}

/* Number of worker threads the oracle runs with. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
