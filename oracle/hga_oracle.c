/*
 * hga_oracle.c -- plain, slow CPU oracle for routed Hierarchical Global
 * Attention (HGA), one layer, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this file.  It shares no code,
 * header, table or helper with the CUDA library and must never be used as a
 * fallback for it.
 *
 * Source of the method: "Long-Context Fine-Tuning with Limited VRAM"
 * (arXiv 2607.15105) as described on three pages:
 *   [TS]  gist.science, "Technical Summary: Long-Context Fine-Tuning with
 *         Limited VRAM", sections 2.1 (HGA: Chunk Selection, Group Selection,
 *         Exact-Token Attention) and 2.2 (Segment-wise Backward and Tiered
 *         Storage);
 *   [PR]  pith.science review of the same paper: "Core claim", "What carries
 *         the argument", Figure 1 and Figure 2 captions, and the
 *         "Axiom & Free-Parameter Ledger" (chunk 64, group 8);
 *   [FA]  the FlashAttention paper cited by the pages (Dao et al., 2022) for
 *         the softmax-attention backward in terms of P, dP and delta.
 *
 * Where the pages leave a step open, the reading taken is stated next to the
 * code (summary = arithmetic mean; block query = mean over the block's
 * queries and the query heads of one KV head; ties go to the lower index;
 * only history chunks are routable; the fixed sink window is the first
 * n_sink history tokens, whole chunks, always attended and never routed; one
 * joint softmax over sink, routed and causal local keys; scale 1/sqrt(D)
 * unless given).
 *
 * Layout of every tensor: contiguous [B, heads, tokens, D] in float64.
 * Arithmetic: float64 throughout, except that the routing functions accept
 * prec == 32, in which case every intermediate of the summaries, block query
 * and scores is rounded to binary32 after each operation, so that the
 * integer routing decision is taken in the same precision as the GPU kernel.
 * (Rounding a float64 result of +, -, * on binary32 operands to binary32
 * gives the correctly rounded binary32 result, so this emulates float math.)
 *
 * Return value of every entry: 0 on success, -1 on an invalid argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double rnd(double x, int prec) { return prec == 32 ? (double)(float)x : x; }

/* ------------------------------------------------------------------------ */
/* Summaries.  [TS] 2.1 "Chunk Selection" / "Group Selection"; [PR] "What    */
/* carries the argument": summaries are built from the model's projected     */
/* keys, one per 64-token chunk and one per 8-token group.  Reading: the     */
/* summary is the arithmetic mean of the keys it covers.                     */
/* ------------------------------------------------------------------------ */

/* out[b,kh,j,:] = (1/span) * sum_{t = span*j .. span*j+span-1} k[b,kh,t,:]
 * Used with span = group size (group summaries) and span = chunk size
 * (chunk summaries: the mean of all keys of the chunk). */
int hgo_span_means(int64_t B, int64_t Hkv, int64_t T, int64_t D, int64_t span,
                   int32_t prec, const double* k, double* out)
{
    if (B < 0 || Hkv < 0 || T < 0 || D <= 0 || span <= 0 || T % span != 0) return -1;
    if (prec != 32 && prec != 64) return -1;
    const int64_t nspan = T / span;
    for (int64_t bh = 0; bh < B * Hkv; ++bh) {
        for (int64_t j = 0; j < nspan; ++j) {
            for (int64_t d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int64_t t = j * span; t < (j + 1) * span; ++t)
                    acc = rnd(acc + k[(bh * T + t) * D + d], prec);
                out[(bh * nspan + j) * D + d] = rnd(acc / (double)span, prec);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Block query.  [TS] 2.1 "Chunk Selection": the current query block scores  */
/* the summaries; [TS] 5 "Causal Leakage" and [PR] referee note on Sec. 6.1: */
/* the routing of a block depends on all query positions in it.  Reading:    */
/* qb[b,kh,n,:] = mean over the G = Hq/Hkv query heads of KV head kh         */
/* (head h belongs to kh = h / G) and over the qblock positions of block n. */
/* ------------------------------------------------------------------------ */
int hgo_block_query(int64_t B, int64_t Hq, int64_t Hkv, int64_t S, int64_t D,
                    int64_t qblock, int32_t prec, const double* q, double* qb)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S < 0 || D <= 0) return -1;
    if (qblock <= 0 || S % qblock != 0 || (prec != 32 && prec != 64)) return -1;
    const int64_t G = Hq / Hkv, nblk = S / qblock;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t kh = 0; kh < Hkv; ++kh)
            for (int64_t n = 0; n < nblk; ++n)
                for (int64_t d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int64_t hh = 0; hh < G; ++hh) {
                        const int64_t h = kh * G + hh;
                        for (int64_t t = n * qblock; t < (n + 1) * qblock; ++t)
                            acc = rnd(acc + q[((b * Hq + h) * S + t) * D + d], prec);
                    }
                    qb[((b * Hkv + kh) * nblk + n) * D + d] =
                        rnd(acc / (double)(G * qblock), prec);
                }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Top-k selection with the lower-index tie rule.                            */
/* ------------------------------------------------------------------------ */
typedef struct { double s; int64_t i; } scored_t;

/* Order: larger score first; equal scores -> lower index first. */
static int by_score_desc_index_asc(const void* pa, const void* pb)
{
    const scored_t* a = (const scored_t*)pa;
    const scored_t* b = (const scored_t*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->i < b->i) ? -1 : (a->i > b->i);
}

static int by_index_asc(const void* pa, const void* pb)
{
    const int64_t a = *(const int64_t*)pa, b = *(const int64_t*)pb;
    return (a < b) ? -1 : (a > b);
}

/* Select the k entries of items[0..n) that come first in the order above,
 * write their ids (items[].i) sorted ascending to sel[0..k), and the gap
 * between the k-th and (k+1)-th score (+inf when k == n) to *gap. */
static int select_topk(scored_t* items, int64_t n, int64_t k, int64_t* sel, double* gap)
{
    if (k < 1 || k > n) return -1;
    qsort(items, (size_t)n, sizeof(scored_t), by_score_desc_index_asc);
    for (int64_t r = 0; r < k; ++r) sel[r] = items[r].i;
    qsort(sel, (size_t)k, sizeof(int64_t), by_index_asc);
    *gap = (k < n) ? items[k - 1].s - items[k].s : INFINITY;
    return 0;
}

/* Exposed for the tests: top-k over a plain score vector. */
int hgo_topk(int64_t n, const double* score, int64_t k, int64_t* sel, double* gap)
{
    if (n < 1) return -1;
    scored_t* items = (scored_t*)malloc((size_t)n * sizeof(scored_t));
    if (!items) return -1;
    for (int64_t i = 0; i < n; ++i) { items[i].s = score[i]; items[i].i = i; }
    int rc = select_topk(items, n, k, sel, gap);
    free(items);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Two-level routing.  [TS] 2.1: "Chunk Selection" scores every closed chunk */
/* summary against the query block and keeps the best chunks; "Group         */
/* Selection" keeps the best groups within the chosen chunks; [PR] Figure 1. */
/* Readings: raw dot-product scores; only history chunks [0, H/chunk) are    */
/* routable (the active segment is covered by the causal local part); group  */
/* selection is one global top-k over all groups of the chosen chunks; ties  */
/* go to the lower index; both index lists are emitted sorted ascending.     */
/*                                                                            */
/* qb  [B,Hkv,nblk,D], gs [B,Hkv,nch*gpc,D], cs [B,Hkv,nch,D]                 */
/* chunk_idx [B,Hkv,nblk,kc], group_idx [B,Hkv,nblk,kg]  (int32)             */
/* chunk_gap, group_gap [B,Hkv,nblk]: score gap at the selection boundary.   */
/* ------------------------------------------------------------------------ */
int hgo_route(int64_t B, int64_t Hkv, int64_t nblk, int64_t D, int64_t nch, int64_t gpc,
              int64_t nsc, int64_t kc, int64_t kg, int32_t prec,
              const double* qb, const double* gs, const double* cs,
              int32_t* chunk_idx, int32_t* group_idx, double* chunk_gap, double* group_gap)
{
    if (B < 0 || Hkv <= 0 || nblk < 0 || D <= 0 || nch < 1 || gpc < 1) return -1;
    if (nsc < 0 || nsc >= nch) return -1;
    if (kc < 1 || kc > nch - nsc || kg < 1 || kg > kc * gpc) return -1;
    if (prec != 32 && prec != 64) return -1;
    const int64_t ngr = nch * gpc;
    scored_t* items = (scored_t*)malloc((size_t)(nch > kc * gpc ? nch : kc * gpc) * sizeof(scored_t));
    int64_t* csel = (int64_t*)malloc((size_t)kc * sizeof(int64_t));
    int64_t* gsel = (int64_t*)malloc((size_t)kg * sizeof(int64_t));
    if (!items || !csel || !gsel) { free(items); free(csel); free(gsel); return -1; }
    int rc = 0;
    for (int64_t bh = 0; bh < B * Hkv && rc == 0; ++bh) {
        for (int64_t n = 0; n < nblk && rc == 0; ++n) {
            const int64_t u = bh * nblk + n;
            const double* qv = qb + u * D;
            /* level 1: every history chunk outside the sink window (the sink's nsc
             * chunks are attended anyway; [TS] 2.1: chunks are selected "alongside
             * fixed sink and local windows") */
            for (int64_t i = nsc; i < nch; ++i) {
                const double* cv = cs + (bh * nch + i) * D;
                double acc = 0.0;
                for (int64_t d = 0; d < D; ++d) acc = rnd(acc + rnd(qv[d] * cv[d], prec), prec);
                items[i - nsc].s = acc;
                items[i - nsc].i = i;
            }
            rc = select_topk(items, nch - nsc, kc, csel, &chunk_gap[u]);
            if (rc) break;
            /* level 2: the gpc groups of every selected chunk */
            int64_t nc = 0;
            for (int64_t c = 0; c < kc; ++c)
                for (int64_t r = 0; r < gpc; ++r) {
                    const int64_t j = csel[c] * gpc + r;
                    const double* gv = gs + (bh * ngr + j) * D;
                    double acc = 0.0;
                    for (int64_t d = 0; d < D; ++d) acc = rnd(acc + rnd(qv[d] * gv[d], prec), prec);
                    items[nc].s = acc;
                    items[nc].i = j;
                    ++nc;
                }
            rc = select_topk(items, nc, kg, gsel, &group_gap[u]);
            if (rc) break;
            for (int64_t c = 0; c < kc; ++c) chunk_idx[u * kc + c] = (int32_t)csel[c];
            for (int64_t r = 0; r < kg; ++r) group_idx[u * kg + r] = (int32_t)gsel[r];
        }
    }
    free(items); free(csel); free(gsel);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Attention.  [TS] 2.1 "Exact-Token Attention": only the exact K/V of the   */
/* selected groups enter attention, summaries never do; [PR] Figure 2: the   */
/* routed tokens come alongside the local window; [TS] 2.2: history K/V are  */
/* detached at the segment boundary, only the active segment is             */
/* differentiable.  Readings: the local window is the whole causal prefix of */
/* the active segment; one joint softmax over routed and local keys.        */
/*                                                                            */
/* Key set of query (b, h, t), t in block n = t / qblock, kh = h / G:         */
/*   the sink window: history tokens 0 .. nsink-1                             */
/*   history tokens group*j .. group*j+group-1 for j in group_idx[b,kh,n,:]  */
/*   active-segment tokens u = 0 .. t                                        */
/* Routed groups never lie in the sink (routing excludes it); a group index  */
/* that does is an invalid argument, as one out of range is.                 */
/* ------------------------------------------------------------------------ */
typedef struct {
    int64_t B, Hq, Hkv, H, S, D, qblock, group, kg, nsink;
    double scale;
    const double *q, *k_hist, *v_hist, *k_seg, *v_seg;
    const int32_t* group_idx;
} layer_t;

/* Pointers to the K and V rows of the key set of row (b, h, t).  Returns the
 * number of keys, nroute = how many of them are history keys (first). */
static int64_t key_set(const layer_t* L, int64_t b, int64_t h, int64_t t,
                       const double** kr, const double** vr, int64_t* nroute)
{
    const int64_t G = L->Hq / L->Hkv, kh = h / G, n = t / L->qblock;
    const int32_t* gi = L->group_idx + ((b * L->Hkv + kh) * (L->S / L->qblock) + n) * L->kg;
    int64_t m = 0;
    for (int64_t pos = 0; pos < L->nsink; ++pos) {
        kr[m] = L->k_hist + ((b * L->Hkv + kh) * L->H + pos) * L->D;
        vr[m] = L->v_hist + ((b * L->Hkv + kh) * L->H + pos) * L->D;
        ++m;
    }
    for (int64_t r = 0; r < L->kg; ++r)
        for (int64_t e = 0; e < L->group; ++e) {
            const int64_t pos = (int64_t)gi[r] * L->group + e;
            kr[m] = L->k_hist + ((b * L->Hkv + kh) * L->H + pos) * L->D;
            vr[m] = L->v_hist + ((b * L->Hkv + kh) * L->H + pos) * L->D;
            ++m;
        }
    *nroute = m;
    for (int64_t u = 0; u <= t; ++u) {
        kr[m] = L->k_seg + ((b * L->Hkv + kh) * L->S + u) * L->D;
        vr[m] = L->v_seg + ((b * L->Hkv + kh) * L->S + u) * L->D;
        ++m;
    }
    return m;
}

static double dot(const double* a, const double* b, int64_t D)
{
    double acc = 0.0;
    for (int64_t d = 0; d < D; ++d) acc += a[d] * b[d];
    return acc;
}

/* Softmax of row (b,h,t) over its key set: fills p[0..m) and returns m;
 * *lse = log sum exp of the scaled scores. */
static int64_t row_softmax(const layer_t* L, int64_t b, int64_t h, int64_t t,
                           const double** kr, const double** vr, double* p, double* lse)
{
    int64_t nroute;
    const int64_t m = key_set(L, b, h, t, kr, vr, &nroute);
    const double* qv = L->q + ((b * L->Hq + h) * L->S + t) * L->D;
    double mx = -INFINITY;
    for (int64_t j = 0; j < m; ++j) {
        p[j] = L->scale * dot(qv, kr[j], L->D);
        if (p[j] > mx) mx = p[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < m; ++j) { p[j] = exp(p[j] - mx); l += p[j]; }
    for (int64_t j = 0; j < m; ++j) p[j] /= l;
    *lse = mx + log(l);
    return m;
}

static int check_layer(const layer_t* L)
{
    if (L->B < 0 || L->Hq <= 0 || L->Hkv <= 0 || L->Hq % L->Hkv) return -1;
    if (L->H < 0 || L->S <= 0 || L->D <= 0 || L->qblock <= 0 || L->S % L->qblock) return -1;
    if (L->group <= 0 || L->H % L->group || L->kg < 0) return -1;
    if (L->nsink < 0 || L->nsink % L->group || L->nsink + L->kg * L->group > L->H) return -1;
    /* every routed group index must name a history group outside the sink */
    const int64_t ngr = L->H / L->group, nsg = L->nsink / L->group;
    const int64_t nidx = L->B * L->Hkv * (L->S / L->qblock) * L->kg;
    for (int64_t i = 0; i < nidx; ++i)
        if (L->group_idx[i] < nsg || L->group_idx[i] >= ngr) return -1;
    return 0;
}

/* Forward.  rows: list of nrows row ids r = (b*Hq + h)*S + t, or NULL for all
 * B*Hq*S rows in order.  o [nrows, D], lse [nrows]. */
int hgo_attn_fwd(int64_t B, int64_t Hq, int64_t Hkv, int64_t H, int64_t S, int64_t D,
                 int64_t qblock, int64_t group, int64_t kg, int64_t nsink, double scale,
                 const double* q, const double* k_hist, const double* v_hist,
                 const double* k_seg, const double* v_seg, const int32_t* group_idx,
                 int64_t nrows, const int64_t* rows, double* o, double* lse)
{
    layer_t L = {B, Hq, Hkv, H, S, D, qblock, group, kg, nsink, scale,
                 q, k_hist, v_hist, k_seg, v_seg, group_idx};
    if (check_layer(&L)) return -1;
    if (!rows) nrows = B * Hq * S;
    const int64_t maxk = nsink + kg * group + S;
    const double** kr = (const double**)malloc((size_t)maxk * sizeof(double*));
    const double** vr = (const double**)malloc((size_t)maxk * sizeof(double*));
    double* p = (double*)malloc((size_t)maxk * sizeof(double));
    if (!kr || !vr || !p) { free(kr); free(vr); free(p); return -1; }
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t r = rows ? rows[i] : i;
        if (r < 0 || r >= B * Hq * S) { free(kr); free(vr); free(p); return -1; }
        const int64_t t = r % S, h = (r / S) % Hq, b = r / (S * Hq);
        const int64_t m = row_softmax(&L, b, h, t, kr, vr, p, &lse[i]);
        for (int64_t d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int64_t j = 0; j < m; ++j) acc += p[j] * vr[j][d];
            o[i * D + d] = acc;
        }
    }
    free(kr); free(vr); free(p);
    return 0;
}

/* Backward ([FA]: dP = dO V^T, delta = rowsum(P o dP), dS = P o (dP - delta),
 * dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO), over the same key sets.
 * Routing is a constant (no gradient, [TS] 2.1) and history K/V are detached
 * ([TS] 2.2), so gradients exist for q and the active-segment k, v only.
 *
 * rows (nrows, or NULL = all): the dq rows to produce, dq [nrows, D].
 * keys (nkeys, or NULL = all B*Hkv*S): active-segment key ids
 *   r = (b*Hkv + kh)*S + u; dk, dv [nkeys, D]. */
int hgo_attn_bwd(int64_t B, int64_t Hq, int64_t Hkv, int64_t H, int64_t S, int64_t D,
                 int64_t qblock, int64_t group, int64_t kg, int64_t nsink, double scale,
                 const double* q, const double* k_hist, const double* v_hist,
                 const double* k_seg, const double* v_seg, const int32_t* group_idx,
                 const double* d_o,
                 int64_t nrows, const int64_t* rows, double* dq,
                 int64_t nkeys, const int64_t* keys, double* dk, double* dv)
{
    layer_t L = {B, Hq, Hkv, H, S, D, qblock, group, kg, nsink, scale,
                 q, k_hist, v_hist, k_seg, v_seg, group_idx};
    if (check_layer(&L)) return -1;
    if (!rows) nrows = B * Hq * S;
    if (!keys) nkeys = B * Hkv * S;
    const int64_t G = Hq / Hkv, maxk = nsink + kg * group + S, nall = B * Hq * S;
    const double** kr = (const double**)malloc((size_t)maxk * sizeof(double*));
    const double** vr = (const double**)malloc((size_t)maxk * sizeof(double*));
    double* p = (double*)malloc((size_t)maxk * sizeof(double));
    double* dp = (double*)malloc((size_t)maxk * sizeof(double));
    /* per-row lse and delta, computed on first use */
    double* row_lse = (double*)malloc((size_t)nall * sizeof(double));
    double* row_delta = (double*)malloc((size_t)nall * sizeof(double));
    char* have = (char*)calloc((size_t)nall, 1);
    int rc = 0;
    if (!kr || !vr || !p || !dp || !row_lse || !row_delta || !have) { rc = -1; goto done; }

    /* dq rows */
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t r = rows ? rows[i] : i;
        if (r < 0 || r >= nall) { rc = -1; goto done; }
        const int64_t t = r % S, h = (r / S) % Hq, b = r / (S * Hq);
        double lse;
        const int64_t m = row_softmax(&L, b, h, t, kr, vr, p, &lse);
        const double* dov = d_o + r * D;
        double delta = 0.0;
        for (int64_t j = 0; j < m; ++j) { dp[j] = dot(dov, vr[j], D); delta += p[j] * dp[j]; }
        for (int64_t d = 0; d < D; ++d) dq[i * D + d] = 0.0;
        for (int64_t j = 0; j < m; ++j) {
            const double ds = p[j] * (dp[j] - delta);
            for (int64_t d = 0; d < D; ++d) dq[i * D + d] += scale * ds * kr[j][d];
        }
    }

    /* dk, dv of active-segment keys: key u is in the key set of every query
     * t >= u of the G query heads of its KV head (causal local part). */
    for (int64_t i = 0; i < nkeys; ++i) {
        const int64_t r = keys ? keys[i] : i;
        if (r < 0 || r >= B * Hkv * S) { rc = -1; goto done; }
        const int64_t u = r % S, kh = (r / S) % Hkv, b = r / (S * Hkv);
        const double* ku = k_seg + r * D;
        const double* vu = v_seg + r * D;
        for (int64_t d = 0; d < D; ++d) { dk[i * D + d] = 0.0; dv[i * D + d] = 0.0; }
        for (int64_t hh = 0; hh < G; ++hh) {
            const int64_t h = kh * G + hh;
            for (int64_t t = u; t < S; ++t) {
                const int64_t row = (b * Hq + h) * S + t;
                const double* qv = q + row * D;
                const double* dov = d_o + row * D;
                if (!have[row]) {
                    const int64_t m = row_softmax(&L, b, h, t, kr, vr, p, &row_lse[row]);
                    double delta = 0.0;
                    for (int64_t j = 0; j < m; ++j) delta += p[j] * dot(dov, vr[j], D);
                    row_delta[row] = delta;
                    have[row] = 1;
                }
                const double pu = exp(scale * dot(qv, ku, D) - row_lse[row]);
                const double ds = pu * (dot(dov, vu, D) - row_delta[row]);
                for (int64_t d = 0; d < D; ++d) {
                    dk[i * D + d] += scale * ds * qv[d];
                    dv[i * D + d] += pu * dov[d];
                }
            }
        }
    }
done:
    free(kr); free(vr); free(p); free(dp); free(row_lse); free(row_delta); free(have);
    return rc;
}
