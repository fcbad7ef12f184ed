/*
 * lca_oracle.c -- plain, slow, double-precision CPU oracle for the
 * Latent-Condensed Attention (LCA) decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker, not the product: only
 * the test suite, the package's smoke entry point and the benchmark's CPU
 * baseline leg may load it.  It shares no code, header, table or helper with
 * the CUDA library under kv_compression_b200/, and includes nothing from it.
 *
 * What it computes follows "Latent-Condensed Transformer for Efficient Long
 * Context Modeling" (gist.science summary of arXiv 2604.12452):
 *   - section 2, the MLA latent is split into a semantic part C_KV (content,
 *     may be pooled) and a positional part K_R (RoPE key, must not be mixed);
 *   - section 2, "O Algoritmo LCA", step 1: the history is cut into contiguous
 *     groups of g tokens while a local window of the w most recent tokens stays
 *     uncompressed;
 *   - step 2: per group, C_KV is pooled with weights taken from the
 *     query-aware attention scores, and the single highest-scoring token of
 *     the group keeps its K_R as the group's positional anchor;
 *   - step 3: attention runs over [condensed groups || window].
 * Section 2 "Vantagens Teoricas": no parameters are added (no bias, no extra
 * scale: the caller folds the softmax scale into the query).
 *
 * The page gives no equations; these readings make it exact (each is listed,
 * with its reason, in the design notes of the repository):
 *   R1 the score used for pooling and for the anchor is the full MLA score
 *      s_t = q_c.c_t + q_r.k_t;
 *   R2 condensation is per head;
 *   R3 the pooling weights are the group-local softmax of s (scale 1);
 *   R4 no +log(g) bias on a condensed entry;
 *   R5 the window is the last w tokens, current token included;
 *   R6 groups start at token 0 and are all full; the (L-w) mod g leftover
 *      tokens join the window: n_G = floor((L-w)/g) if L > w, else 0;
 *   R7 the anchor is the lowest index attaining the group maximum;
 *   R8 the value of a condensed entry is its pooled latent c_bar (absorbed
 *      MLA: the value is the latent itself).
 *
 * Two formulations are implemented:
 *   A (returned): materialise every condensed entry (c_bar_j, k_{a_j}),
 *     form the logits of [condensed || window] from the entry vectors, and
 *     take a textbook two-pass softmax-weighted sum of the entry values;
 *   B (cross-check): the folded form, S_j = sum_t w_t sc_t + sr_{a_j}, the
 *     per-token weight p_j w_t, never forming c_bar_j as a logit operand.
 * Both are plain restatements; tests pin A against closed forms, library
 * attention and brute force, and check B against A.
 *
 * Element types: 0 = float32, 1 = bfloat16 stored as uint16 (exact widening:
 * the 16 bits are the top half of the float32 pattern).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F32 0
#define ORACLE_BF16 1

static double elem(const void *p, int64_t i, int dtype)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)p)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Dot product of a double query with row `row` (length n) of a stored matrix. */
static double dot_row(const double *q, const void *mat, int64_t row, int n, int dtype)
{
    double acc = 0.0;
    for (int i = 0; i < n; ++i)
        acc += q[i] * elem(mat, row * (int64_t)n + i, dtype);
    return acc;
}

int64_t lca_oracle_num_groups(int64_t L, int g, int w)
{
    /* Reading R6: full groups from position 0, leftovers join the window. */
    if (g < 1 || w < 0 || L <= (int64_t)w)
        return 0;
    return (L - (int64_t)w) / g;
}

/* Per-head scratch: scores and per-group softmax statistics. */
typedef struct {
    double *qc, *qr;        /* query of this head, widened */
    double *sc, *sr, *s;    /* semantic, positional and full score per token */
    double *gmax, *gden;    /* per group: max score and sum of exp(s - max) */
    int32_t *ganc;          /* per group: anchor (absolute position) */
    double *ell;            /* logits of the entries [condensed || window] */
    double *cbar;           /* one pooled latent */
} scratch_t;

static int scratch_alloc(scratch_t *w, int d_c, int d_r, int64_t L, int64_t nG)
{
    int64_t ne = nG + L; /* upper bound on the number of entries */
    w->qc = malloc(sizeof(double) * (size_t)d_c);
    w->qr = malloc(sizeof(double) * (size_t)(d_r > 0 ? d_r : 1));
    w->sc = malloc(sizeof(double) * (size_t)L);
    w->sr = malloc(sizeof(double) * (size_t)L);
    w->s = malloc(sizeof(double) * (size_t)L);
    w->gmax = malloc(sizeof(double) * (size_t)(nG > 0 ? nG : 1));
    w->gden = malloc(sizeof(double) * (size_t)(nG > 0 ? nG : 1));
    w->ganc = malloc(sizeof(int32_t) * (size_t)(nG > 0 ? nG : 1));
    w->ell = malloc(sizeof(double) * (size_t)ne);
    w->cbar = malloc(sizeof(double) * (size_t)d_c);
    return (w->qc && w->qr && w->sc && w->sr && w->s && w->gmax && w->gden &&
            w->ganc && w->ell && w->cbar) ? 0 : -1;
}

static void scratch_free(scratch_t *w)
{
    free(w->qc); free(w->qr); free(w->sc); free(w->sr); free(w->s);
    free(w->gmax); free(w->gden); free(w->ganc); free(w->ell); free(w->cbar);
}

/*
 * Step 2 pooling weight of token t of group j: the group-local softmax of the
 * full score (readings R1, R3).
 */
static double pool_weight(const scratch_t *w, int64_t j, int64_t t)
{
    return exp(w->s[t] - w->gmax[j]) / w->gden[j];
}

/* c_bar_j = sum_{t in G_j} w_t c_t  (reading R8: the condensed value). */
static void pooled_latent(const scratch_t *w, const void *c_kv, int d_c, int dtype,
                          int g, int64_t j, double *cbar)
{
    for (int i = 0; i < d_c; ++i)
        cbar[i] = 0.0;
    for (int64_t t = j * g; t < (j + 1) * g; ++t) {
        double wt = pool_weight(w, j, t);
        for (int i = 0; i < d_c; ++i)
            cbar[i] += wt * elem(c_kv, t * (int64_t)d_c + i, dtype);
    }
}

/*
 * One (sequence, head): q_c [d_c], q_r [d_r]; c_kv [L][d_c]; k_r [L][d_r].
 * Writes out [d_c] (formulation A or B), anchor [n_G], and optionally the
 * top-2 score gap per group and max |s| over the sequence.
 */
static void lca_one_head(int d_c, int d_r, int64_t L, int g, int w_win, int dtype,
                         const void *q_c, const void *q_r, const void *c_kv, const void *k_r,
                         int formulation, double *out, int32_t *anchor, double *tie_gap,
                         double *max_abs_s, scratch_t *w)
{
    const int64_t nG = lca_oracle_num_groups(L, g, w_win);
    const int64_t win0 = nG * g; /* first window token */

    for (int i = 0; i < d_c; ++i) w->qc[i] = elem(q_c, i, dtype);
    for (int i = 0; i < d_r; ++i) w->qr[i] = elem(q_r, i, dtype);

    /* Scores of every cached token (section 1: MLA attends over all latents). */
    double amax = 0.0;
    for (int64_t t = 0; t < L; ++t) {
        w->sc[t] = dot_row(w->qc, c_kv, t, d_c, dtype);
        w->sr[t] = dot_row(w->qr, k_r, t, d_r, dtype);
        w->s[t] = w->sc[t] + w->sr[t];
        if (fabs(w->s[t]) > amax) amax = fabs(w->s[t]);
    }
    if (max_abs_s) *max_abs_s = amax;

    /* Step 1 + 2: groups, group-local softmax statistics, anchors. */
    for (int64_t j = 0; j < nG; ++j) {
        int64_t t0 = j * g;
        double m = w->s[t0];
        int64_t a = t0;
        for (int64_t t = t0 + 1; t < t0 + g; ++t) {
            if (w->s[t] > m) { m = w->s[t]; a = t; } /* strict: lowest index wins ties (R7) */
        }
        double second = -INFINITY;
        for (int64_t t = t0; t < t0 + g; ++t)
            if (t != a && w->s[t] > second) second = w->s[t];
        double den = 0.0;
        for (int64_t t = t0; t < t0 + g; ++t) den += exp(w->s[t] - m);
        w->gmax[j] = m;
        w->gden[j] = den;
        w->ganc[j] = (int32_t)a;
        if (anchor) anchor[j] = (int32_t)a;
        if (tie_gap) tie_gap[j] = (g > 1) ? (m - second) : INFINITY;
    }

    const int64_t nE = nG + (L - win0); /* entries: condensed groups, then window */

    if (formulation == 0) {
        /* ---- Formulation A: materialised condensed entries, textbook softmax. */
        /* Pass 1: logit of each entry, q . [value; positional key]. */
        for (int64_t j = 0; j < nG; ++j) {
            pooled_latent(w, c_kv, d_c, dtype, g, j, w->cbar);
            double l = 0.0;
            for (int i = 0; i < d_c; ++i) l += w->qc[i] * w->cbar[i];
            l += dot_row(w->qr, k_r, w->ganc[j], d_r, dtype); /* anchor's K_R */
            w->ell[j] = l;
        }
        for (int64_t t = win0; t < L; ++t)
            w->ell[nG + (t - win0)] = dot_row(w->qc, c_kv, t, d_c, dtype) +
                                      dot_row(w->qr, k_r, t, d_r, dtype);
        double M = -INFINITY;
        for (int64_t e = 0; e < nE; ++e) if (w->ell[e] > M) M = w->ell[e];
        double Z = 0.0;
        for (int64_t e = 0; e < nE; ++e) Z += exp(w->ell[e] - M);
        /* Pass 2: softmax-weighted sum of the entry values. */
        for (int i = 0; i < d_c; ++i) out[i] = 0.0;
        for (int64_t j = 0; j < nG; ++j) {
            double p = exp(w->ell[j] - M) / Z;
            pooled_latent(w, c_kv, d_c, dtype, g, j, w->cbar);
            for (int i = 0; i < d_c; ++i) out[i] += p * w->cbar[i];
        }
        for (int64_t t = win0; t < L; ++t) {
            double p = exp(w->ell[nG + (t - win0)] - M) / Z;
            for (int i = 0; i < d_c; ++i) out[i] += p * elem(c_kv, t * (int64_t)d_c + i, dtype);
        }
    } else {
        /* ---- Formulation B: folded; q_c . c_bar_j = sum_t w_t (q_c . c_t). */
        for (int64_t j = 0; j < nG; ++j) {
            double S = 0.0;
            for (int64_t t = j * g; t < (j + 1) * g; ++t) S += pool_weight(w, j, t) * w->sc[t];
            w->ell[j] = S + w->sr[w->ganc[j]];
        }
        for (int64_t t = win0; t < L; ++t) w->ell[nG + (t - win0)] = w->s[t];
        double M = -INFINITY;
        for (int64_t e = 0; e < nE; ++e) if (w->ell[e] > M) M = w->ell[e];
        double Z = 0.0;
        for (int64_t e = 0; e < nE; ++e) Z += exp(w->ell[e] - M);
        for (int i = 0; i < d_c; ++i) out[i] = 0.0;
        for (int64_t j = 0; j < nG; ++j) {
            double pj = exp(w->ell[j] - M);
            for (int64_t t = j * g; t < (j + 1) * g; ++t) {
                double pt = pj * pool_weight(w, j, t); /* group weight x in-group weight */
                for (int i = 0; i < d_c; ++i) out[i] += pt * elem(c_kv, t * (int64_t)d_c + i, dtype);
            }
        }
        for (int64_t t = win0; t < L; ++t) {
            double pt = exp(w->ell[nG + (t - win0)] - M);
            for (int i = 0; i < d_c; ++i) out[i] += pt * elem(c_kv, t * (int64_t)d_c + i, dtype);
        }
        for (int i = 0; i < d_c; ++i) out[i] /= Z;
    }
}

/*
 * LCA decode for one sequence, all H heads.
 *   q_c [H][d_c], q_r [H][d_r], c_kv [L][d_c], k_r [L][d_r] in `dtype`;
 *   out [H][d_c] (double); anchor [H][n_G] int32 absolute positions (may be
 *   NULL when n_G == 0); tie_gap [H][n_G] and max_abs_s [H] optional (NULL).
 *   formulation: 0 = A (materialised), 1 = B (folded).
 *   nthreads: OpenMP threads over heads (0 = runtime default).
 * Returns 0, or -1 on invalid arguments, -2 when scratch cannot be allocated.
 */
int lca_oracle_seq(int H, int d_c, int d_r, int64_t L, int g, int w_win, int dtype,
                   const void *q_c, const void *q_r, const void *c_kv, const void *k_r,
                   int formulation, double *out, int32_t *anchor, double *tie_gap,
                   double *max_abs_s, int nthreads)
{
    if (H < 1 || d_c < 1 || d_r < 0 || L < 1 || g < 1 || w_win < 0 ||
        (dtype != ORACLE_F32 && dtype != ORACLE_BF16) || !q_c || !c_kv || !out ||
        (d_r > 0 && (!q_r || !k_r)))
        return -1;
    const int64_t nG = lca_oracle_num_groups(L, g, w_win);
    if (nG > 0 && !anchor)
        return -1;
    int status = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        scratch_t w;
        int ok = scratch_alloc(&w, d_c, d_r, L, nG) == 0;
        if (!ok) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = -2;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int h = 0; h < H; ++h) {
            if (!ok) continue;
            const size_t esz = dtype == ORACLE_F32 ? 4 : 2;
            lca_one_head(d_c, d_r, L, g, w_win, dtype,
                         (const char *)q_c + (size_t)h * d_c * esz,
                         d_r > 0 ? (const char *)q_r + (size_t)h * d_r * esz : NULL,
                         c_kv, k_r, formulation, out + (size_t)h * d_c,
                         anchor ? anchor + (size_t)h * nG : NULL,
                         tie_gap ? tie_gap + (size_t)h * nG : NULL,
                         max_abs_s ? max_abs_s + h : NULL, &w);
        }
        scratch_free(&w);
    }
    return status;
}

/*
 * Dense MLA decode for one sequence (section 1: MLA attends densely over all
 * latent tokens): out = sum_t softmax(s)_t c_t, textbook two-pass softmax.
 */
int mla_oracle_seq(int H, int d_c, int d_r, int64_t L, int dtype,
                   const void *q_c, const void *q_r, const void *c_kv, const void *k_r,
                   double *out, int nthreads)
{
    if (H < 1 || d_c < 1 || d_r < 0 || L < 1 || (dtype != ORACLE_F32 && dtype != ORACLE_BF16) ||
        !q_c || !c_kv || !out || (d_r > 0 && (!q_r || !k_r)))
        return -1;
    int status = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double *qc = malloc(sizeof(double) * (size_t)d_c);
        double *qr = malloc(sizeof(double) * (size_t)(d_r > 0 ? d_r : 1));
        double *s = malloc(sizeof(double) * (size_t)L);
        int ok = qc && qr && s;
        if (!ok) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = -2;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int h = 0; h < H; ++h) {
            if (!ok) continue;
            const size_t esz = dtype == ORACLE_F32 ? 4 : 2;
            const void *qch = (const char *)q_c + (size_t)h * d_c * esz;
            const void *qrh = d_r > 0 ? (const char *)q_r + (size_t)h * d_r * esz : NULL;
            for (int i = 0; i < d_c; ++i) qc[i] = elem(qch, i, dtype);
            for (int i = 0; i < d_r; ++i) qr[i] = elem(qrh, i, dtype);
            double M = -INFINITY;
            for (int64_t t = 0; t < L; ++t) {
                s[t] = dot_row(qc, c_kv, t, d_c, dtype) + dot_row(qr, k_r, t, d_r, dtype);
                if (s[t] > M) M = s[t];
            }
            double Z = 0.0;
            for (int64_t t = 0; t < L; ++t) Z += exp(s[t] - M);
            double *o = out + (size_t)h * d_c;
            for (int i = 0; i < d_c; ++i) o[i] = 0.0;
            for (int64_t t = 0; t < L; ++t) {
                double p = exp(s[t] - M) / Z;
                for (int i = 0; i < d_c; ++i) o[i] += p * elem(c_kv, t * (int64_t)d_c + i, dtype);
            }
        }
        free(qc); free(qr); free(s);
    }
    return status;
}

/*
 * Stored, head-shared condensed cache.  The page's memory and decode-latency
 * gains (section 4, "Eficiencia": the KV cache at 128K shrinks by ~90%, decode
 * latency per token drops 1.8x) come from keeping the condensed groups
 * instead of the tokens they stand for.  A stored entry cannot depend on the
 * queries of later steps, so a group is condensed once, with the query of
 * the step that condenses it, and one entry serves every head.  The page does
 * not say how the heads' scores are combined; the reading here is the plain
 * mean over heads:
 *   s_bar_t = (1/H) sum_h (q_c^h . c_t + q_r^h . k_t)
 *   w_t = softmax_{t in G_j}(s_bar_t),  a_j = lowest t with the largest s_bar_t,
 *   stored entry j = (c_bar_j = sum_t w_t c_t,  k_{a_j}).
 * Decode over the stored cache is plain softmax attention (value = latent) over
 * [stored condensed entries || window tokens]; an optional bias b is added to
 * the condensed entries' logits (b = log g treats an entry as the g tokens it
 * stands for; the page names no bias, so the default is 0).
 */

/*
 * Condense groups j0 .. j0+n-1 of one sequence (tokens [j g, j g + g), all
 * below L) with the head-mean score of the query q_c [H][d_c], q_r [H][d_r].
 * Writes cbar [n][d_c], kanc [n][d_r] (doubles), anchor [n] (absolute
 * positions) and optionally tie_gap [n] (top-2 gap of s_bar per group, +inf
 * for g = 1) and max_abs [1] (max |s_bar| over the condensed tokens).
 * Returns 0, -1 on invalid arguments, -2 when scratch cannot be allocated.
 */
int lca_oracle_condense_shared(int H, int d_c, int d_r, int64_t L, int g, int64_t j0, int64_t n,
                               int dtype, const void *q_c, const void *q_r, const void *c_kv,
                               const void *k_r, double *cbar, double *kanc, int32_t *anchor,
                               double *tie_gap, double *max_abs)
{
    if (H < 1 || d_c < 1 || d_r < 0 || L < 1 || g < 1 || j0 < 0 || n < 0 ||
        (j0 + n) * (int64_t)g > L || (dtype != ORACLE_F32 && dtype != ORACLE_BF16) ||
        !q_c || !c_kv || !cbar || !anchor || (d_r > 0 && (!q_r || !k_r || !kanc)))
        return -1;
    double *qc = malloc(sizeof(double) * (size_t)d_c);
    double *qr = malloc(sizeof(double) * (size_t)(d_r > 0 ? d_r : 1));
    double *sbar = malloc(sizeof(double) * (size_t)g);
    if (!qc || !qr || !sbar) {
        free(qc); free(qr); free(sbar);
        return -2;
    }
    const size_t esz = dtype == ORACLE_F32 ? 4 : 2;
    double amax = 0.0;
    for (int64_t jj = 0; jj < n; ++jj) {
        const int64_t t0 = (j0 + jj) * g;
        for (int u = 0; u < g; ++u) sbar[u] = 0.0;
        /* per-head scores, then their mean */
        for (int h = 0; h < H; ++h) {
            for (int i = 0; i < d_c; ++i) qc[i] = elem((const char *)q_c + (size_t)h * d_c * esz, i, dtype);
            for (int i = 0; i < d_r; ++i) qr[i] = elem((const char *)q_r + (size_t)h * d_r * esz, i, dtype);
            for (int u = 0; u < g; ++u)
                sbar[u] += dot_row(qc, c_kv, t0 + u, d_c, dtype) + dot_row(qr, k_r, t0 + u, d_r, dtype);
        }
        for (int u = 0; u < g; ++u) {
            sbar[u] /= (double)H;
            if (fabs(sbar[u]) > amax) amax = fabs(sbar[u]);
        }
        double m = sbar[0];
        int a = 0;
        for (int u = 1; u < g; ++u)
            if (sbar[u] > m) { m = sbar[u]; a = u; }   /* strict: lowest index wins ties */
        double second = -INFINITY, den = 0.0;
        for (int u = 0; u < g; ++u) {
            if (u != a && sbar[u] > second) second = sbar[u];
            den += exp(sbar[u] - m);
        }
        double *cb = cbar + jj * (int64_t)d_c;
        for (int i = 0; i < d_c; ++i) cb[i] = 0.0;
        for (int u = 0; u < g; ++u) {
            const double wt = exp(sbar[u] - m) / den;
            for (int i = 0; i < d_c; ++i) cb[i] += wt * elem(c_kv, (t0 + u) * (int64_t)d_c + i, dtype);
        }
        for (int i = 0; i < d_r; ++i) kanc[jj * (int64_t)d_r + i] = elem(k_r, (t0 + a) * (int64_t)d_r + i, dtype);
        anchor[jj] = (int32_t)(t0 + a);
        if (tie_gap) tie_gap[jj] = g > 1 ? m - second : INFINITY;
    }
    if (max_abs) *max_abs = amax;
    free(qc); free(qr); free(sbar);
    return 0;
}

/*
 * Decode one sequence over a stored cache: n_cond condensed entries (cbar
 * [n_cond][d_c], kanc [n_cond][d_r], doubles) followed by n_win window tokens
 * (c_win [n_win][d_c], k_win [n_win][d_r] in `dtype`), for every head of q.
 * logit_e = q_c . c_e + q_r . k_e (+ bias for a condensed entry); out [H][d_c] =
 * sum_e softmax(logit)_e c_e, textbook two-pass softmax.  Returns 0 or -1/-2.
 */
int lca_oracle_decode_stored(int H, int d_c, int d_r, int64_t n_cond, int64_t n_win, int dtype,
                             const void *q_c, const void *q_r, const double *cbar,
                             const double *kanc, const void *c_win, const void *k_win,
                             double bias, double *out)
{
    const int64_t nE = n_cond + n_win;
    if (H < 1 || d_c < 1 || d_r < 0 || n_cond < 0 || n_win < 0 || nE < 1 ||
        (dtype != ORACLE_F32 && dtype != ORACLE_BF16) || !q_c || !out ||
        (n_cond > 0 && (!cbar || (d_r > 0 && !kanc))) || (n_win > 0 && (!c_win || (d_r > 0 && !k_win))) ||
        (d_r > 0 && !q_r))
        return -1;
    double *qc = malloc(sizeof(double) * (size_t)d_c);
    double *qr = malloc(sizeof(double) * (size_t)(d_r > 0 ? d_r : 1));
    double *ell = malloc(sizeof(double) * (size_t)nE);
    if (!qc || !qr || !ell) {
        free(qc); free(qr); free(ell);
        return -2;
    }
    const size_t esz = dtype == ORACLE_F32 ? 4 : 2;
    for (int h = 0; h < H; ++h) {
        for (int i = 0; i < d_c; ++i) qc[i] = elem((const char *)q_c + (size_t)h * d_c * esz, i, dtype);
        for (int i = 0; i < d_r; ++i) qr[i] = elem((const char *)q_r + (size_t)h * d_r * esz, i, dtype);
        for (int64_t e = 0; e < n_cond; ++e) {
            double l = bias;
            for (int i = 0; i < d_c; ++i) l += qc[i] * cbar[e * (int64_t)d_c + i];
            for (int i = 0; i < d_r; ++i) l += qr[i] * kanc[e * (int64_t)d_r + i];
            ell[e] = l;
        }
        for (int64_t t = 0; t < n_win; ++t)
            ell[n_cond + t] = dot_row(qc, c_win, t, d_c, dtype) + dot_row(qr, k_win, t, d_r, dtype);
        double M = -INFINITY;
        for (int64_t e = 0; e < nE; ++e) if (ell[e] > M) M = ell[e];
        double Z = 0.0;
        for (int64_t e = 0; e < nE; ++e) Z += exp(ell[e] - M);
        double *o = out + (size_t)h * d_c;
        for (int i = 0; i < d_c; ++i) o[i] = 0.0;
        for (int64_t e = 0; e < n_cond; ++e) {
            const double pe = exp(ell[e] - M) / Z;
            for (int i = 0; i < d_c; ++i) o[i] += pe * cbar[e * (int64_t)d_c + i];
        }
        for (int64_t t = 0; t < n_win; ++t) {
            const double pe = exp(ell[n_cond + t] - M) / Z;
            for (int i = 0; i < d_c; ++i) o[i] += pe * elem(c_win, t * (int64_t)d_c + i, dtype);
        }
    }
    free(qc); free(qr); free(ell);
    return 0;
}

/*
 * Context sharding: the entries of one sequence ([condensed groups || window],
 * section 2 steps 1-3 for the whole context of L_total tokens) are split by
 * position among several holders -- one slice of tokens [pos0, pos0 + n_tok)
 * each, cut on group boundaries inside the condensed part -- and each holder
 * computes the partial softmax sums of the entries it holds:
 *   M = max_e logit_e,  Z = sum_e exp(logit_e - M),  O = sum_e exp(logit_e - M) value_e,
 * over its condensed groups (all g tokens inside the slice) and window tokens.
 * The partials merge exactly (the online-softmax merge of the Pulsar Attention
 * page, "Fase 2"): M* = max M_i, out = sum_i e^{M_i - M*} O_i / sum_i e^{M_i - M*} Z_i.
 * An empty slice gives M = -inf, Z = 0, O = 0.
 *
 * One (sequence, head): the whole cache c_kv [L_total][d_c], k_r [L_total][d_r]
 * is passed and only rows of the slice are read.  Writes m [1], z [1], o [d_c]
 * and the anchors of the slice's groups (anchor [n_slice_groups], absolute).
 * Returns 0, -1 when the slice cuts a group, -2 on allocation failure.
 */
int lca_oracle_partial(int d_c, int d_r, int64_t L_total, int g, int w_win, int64_t pos0,
                       int64_t n_tok, int dtype, const void *q_c, const void *q_r,
                       const void *c_kv, const void *k_r, double *m, double *z, double *o,
                       int32_t *anchor)
{
    const int64_t nG = lca_oracle_num_groups(L_total, g, w_win);
    const int64_t win0 = nG * g;
    const int64_t end = pos0 + n_tok;
    if (pos0 < 0 || n_tok < 0 || end > L_total || g < 1 ||
        (pos0 < win0 && pos0 % g != 0) || (end < win0 && end % g != 0))
        return -1;
    scratch_t w;
    if (scratch_alloc(&w, d_c, d_r, L_total, nG) != 0) {
        scratch_free(&w);
        return -2;
    }
    for (int i = 0; i < d_c; ++i) w.qc[i] = elem(q_c, i, dtype);
    for (int i = 0; i < d_r; ++i) w.qr[i] = elem(q_r, i, dtype);
    /* scores of the slice's tokens only */
    for (int64_t t = pos0; t < end; ++t) {
        w.sc[t] = dot_row(w.qc, c_kv, t, d_c, dtype);
        w.sr[t] = dot_row(w.qr, k_r, t, d_r, dtype);
        w.s[t] = w.sc[t] + w.sr[t];
    }
    const int64_t j_lo = pos0 < win0 ? pos0 / g : nG;          /* groups inside the slice */
    const int64_t j_hi = end < win0 ? end / g : nG;
    int64_t ne = 0;
    for (int64_t j = j_lo; j < j_hi; ++j) {                      /* step 2 per group */
        const int64_t t0 = j * g;
        double mx = w.s[t0];
        int64_t a = t0;
        for (int64_t t = t0 + 1; t < t0 + g; ++t)
            if (w.s[t] > mx) { mx = w.s[t]; a = t; }
        double den = 0.0;
        for (int64_t t = t0; t < t0 + g; ++t) den += exp(w.s[t] - mx);
        w.gmax[j] = mx;
        w.gden[j] = den;
        w.ganc[j] = (int32_t)a;
        if (anchor) anchor[j - j_lo] = (int32_t)a;
        pooled_latent(&w, c_kv, d_c, dtype, g, j, w.cbar);
        double l = 0.0;
        for (int i = 0; i < d_c; ++i) l += w.qc[i] * w.cbar[i];
        w.ell[ne++] = l + dot_row(w.qr, k_r, a, d_r, dtype);
    }
    const int64_t wlo = pos0 > win0 ? pos0 : win0;               /* window tokens inside */
    for (int64_t t = wlo; t < end; ++t) w.ell[ne++] = w.s[t];
    double M = -INFINITY;
    for (int64_t e = 0; e < ne; ++e) if (w.ell[e] > M) M = w.ell[e];
    double Z = 0.0;
    for (int i = 0; i < d_c; ++i) o[i] = 0.0;
    int64_t e = 0;
    for (int64_t j = j_lo; j < j_hi; ++j, ++e) {
        const double p = exp(w.ell[e] - M);
        Z += p;
        pooled_latent(&w, c_kv, d_c, dtype, g, j, w.cbar);
        for (int i = 0; i < d_c; ++i) o[i] += p * w.cbar[i];
    }
    for (int64_t t = wlo; t < end; ++t, ++e) {
        const double p = exp(w.ell[e] - M);
        Z += p;
        for (int i = 0; i < d_c; ++i) o[i] += p * elem(c_kv, t * (int64_t)d_c + i, dtype);
    }
    *m = M;
    *z = Z;
    scratch_free(&w);
    return 0;
}

/* Merge n partials (m [n], z [n], o [n][d_c]) into out [d_c]. */
void lca_oracle_merge(int n, int d_c, const double *m, const double *z, const double *o, double *out)
{
    double M = -INFINITY;
    for (int i = 0; i < n; ++i) if (m[i] > M) M = m[i];
    double Z = 0.0;
    for (int k = 0; k < d_c; ++k) out[k] = 0.0;
    for (int i = 0; i < n; ++i) {
        if (m[i] == -INFINITY) continue;                         /* an empty slice */
        const double f = exp(m[i] - M);
        Z += f * z[i];
        for (int k = 0; k < d_c; ++k) out[k] += f * o[(int64_t)i * d_c + k];
    }
    for (int k = 0; k < d_c; ++k) out[k] /= Z;
}
