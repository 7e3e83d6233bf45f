/*
 * gm_oracle.c - CPU oracle of the Graph Machine sparse layer: sparse edge referral (SER),
 * sparse edge attention (SEA), and the backward passes of both.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline leg load this library; the CUDA library shares no code with it and never
 * calls it. It is written to be checked against the method's description by eye: plain
 * loops, one output row at a time, no blocking, no fusion, no reordering. The referral step
 * runs in fp32 because its rounding decides which edges survive; attention and its backward
 * run in fp64 on inputs widened exactly from fp32/bf16.
 *
 * Source: "Graph Machine: Towards Better Pretraining via Edges" (arXiv 2609.02881), as
 * summarised on ai.info:
 *   [KC2]  "Key Contributions", item 2: edge state = integer indices plus fp weights,
 *          shape n x k x s1 per sequence.
 *   [KC3]  "Key Contributions", item 3: SER composes two-hop paths, A' = Sparsify_s1(A1 A2),
 *          cutting the up-to s2*s3 candidates back to s1; SEA picks the K/V positions by the
 *          edge indices and combines the scaled query-key score with the log edge weight as
 *          a product of experts.
 *   [MPE2] "Methodology in Plain English", paragraph on referral: the first leg's indices
 *          fetch the second leg's indices and weights, two-hop paths become one-hop edges,
 *          hard top-s selection keeps the budget; only kept weights carry gradient.
 *   [MPE3] same section, paragraph on SEA: a handful of K/V positions per edge set, weight
 *          = scaled q.k + log(mixed edge weight), no RoPE.
 *   [MPE4] same section, hybrid paragraph: a padding token at the start of each sequence
 *          absorbs underflowing edge indices.
 *   [MF4]  "Main Findings", bullet on more edges: the cross-edge mixing is full (every stored
 *          channel feeds every leg channel), so its cost grows as k^2.
 *   [MF5]  "Main Findings", bullet on refresh and realignment: refresh edges help; same
 *          section as [MPE2], last sentence: refresh edges come from the input edges or from
 *          the top positions of the latest dense attention layer.
 *
 * Readings where the pages are silent (the CUDA library applies the same ones):
 *   R1  A1 and A2 share the edge channel h (leg mixing happens upstream).
 *   R2  candidate c = a*s3 + e has weight fl32(w1[a] * w2[e]); duplicates of a target are
 *       summed in fp32, each add rounded to nearest, in ascending c, starting from the first.
 *   R3  a slot is active iff its weight is > 0. Inactive slots are never dereferenced.
 *       Zero-weight candidates are dropped before the merge.
 *   R4  top-s1 order: larger merged weight first, then smaller index; outputs stored in that
 *       order; missing slots padded with (index 0, weight 0.0f) - the padding token.
 *   R5  no renormalisation after top-s1.
 *   R6  SEA: z_j = scale * <q, K[t_j]> + ln w_j over active slots j; softmax over them;
 *       o = sum p_j V[t_j]; lse = max z + ln sum exp(z - max z); a row with no active slot
 *       gives o = 0 and lse = -inf. Duplicate indices in a row count as separate slots.
 *   R7  GQA: query head hq reads KV head hq / (Hq / Hkv) (contiguous groups).
 *   R8  an active slot whose index lies outside [0, n) is skipped and counted; the count is
 *       the return value of each entry point.
 *   R9  SER backward: only the kept (top-s1, weight > 0) merged weights carry gradient; the
 *       selection itself is piecewise constant and passes none; indices get none.
 *   R10 leg mixing: leg L (L = 1, 2) of edge channel h at token (b, i) takes every stored edge
 *       (c, a) of that token - all k channels c, all s0 slots a - as a candidate with target
 *       E.idx[b,i,c,a] and weight fl32(M_L[b,i,h,c] * E.w[b,i,c,a]), in ascending c*s0 + a.
 *       The mixing coefficients M_L >= 0 are inputs (how they are computed from the node
 *       features is upstream); one [k, k] matrix shared by all tokens is the case of a zero
 *       token stride.
 *   R11 each leg is then merged, ordered and cut to its budget (s2 for leg 1, s3 for leg 2)
 *       exactly as SER's steps (R2-R5): the "sparsify" of both steps is one operation.
 *   R12 leg backward: as R9, only the kept merged leg weights carry gradient, to both the
 *       stored weights and the mixing coefficients. Each kept weight is differentiated as the
 *       sum over the active stored edges that reach its target of coefficient x weight, so an
 *       active edge whose product was zero (a zero coefficient) still passes the gradient of
 *       its coefficient: R3's dropping of zero products shapes the forward's candidate set,
 *       not the derivative. The gradient of the coefficients is returned per token,
 *       [B, n, k, k], also when they were shared (the caller sums it).
 *   R13 refresh edges: a set F of extra edges per (b, i, h) (the original input edges, or the
 *       top positions of a dense attention layer, produced upstream) joins the referral's
 *       candidates after the s2*s3 two-hop paths, with its own weights: A' =
 *       Sparsify_s1(A1 A2 + F). Candidate order: the paths in ascending c = a*s3 + e, then
 *       the refresh slots in ascending f; merge, order and cut as R2-R5. A kept target's
 *       merged weight passes its gradient unchanged to every refresh slot that reaches it.
 *   R14 the dense layer whose top positions give refresh edges is plain causal softmax
 *       attention: query head hq of token i gives position t <= i the probability
 *       P[hq](i, t) = exp(scale <q[i,hq], k[t,h]> - lse[i,hq]), h = hq / (Hq / Hkv), where
 *       lse[i,hq] is the natural-log normaliser of that row, as the dense layer's forward
 *       returns it (oracle_dense_lse computes it from the definition).
 *   R15 the refresh edges of (b, i, h) are the sf positions t <= i with the largest attention
 *       mass of KV head h: the mean of P[hq](i, t) over the query heads hq of its group. The
 *       edge weight is that mean (computed in fp64, rounded to fp32); ties go to the smaller
 *       position; rows with fewer than sf positions (i + 1 < sf) are padded with (index 0,
 *       weight 0.0f); the slots are ordered by mass descending, then position ascending.
 *
 * Layouts are contiguous row-major: features [B, n, H, d], edges [B, n, k, s].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_MAX_CAND 1024

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the parallel loops from now on (the benchmark times the oracle on one core and on
 * all of them). */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    omp_set_num_threads(n > 0 ? n : 1);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------------------------------
 * SER: A' = Sparsify_s1(A1 A2)   [KC3], [MPE2]; readings R1-R5, R8.
 *
 * For each (b, i, h): every candidate two-hop path i -> j = A1.idx[a] -> t = A2[j].idx[e]
 * has weight A1.w[a] * A2[j].w[e]; paths that reach the same t are summed (the product of
 * the two sparse adjacency matrices restricted to its support), and the s1 heaviest targets
 * are kept.
 * ---------------------------------------------------------------------------------------- */
int64_t oracle_ser(const int32_t *a1_idx, const float *a1_w, int s2,
                   const int32_t *a2_idx, const float *a2_w, int s3,
                   int32_t *out_idx, float *out_w, int s1,
                   int B, int n, int k)
{
    const int64_t rows = (int64_t)B * n * k;
    int64_t bad = 0;
    if (s2 * s3 > ORACLE_MAX_CAND) return -1;

#pragma omp parallel for schedule(static) reduction(+ : bad)
    for (int64_t row = 0; row < rows; ++row) {
        const int h = (int)(row % k);
        const int64_t b = row / ((int64_t)n * k);

        /* 1. candidates in ascending c = a*s3 + e */
        int32_t cand_t[ORACLE_MAX_CAND];
        float cand_u[ORACLE_MAX_CAND];
        int nc = 0;
        for (int a = 0; a < s2; ++a) {
            const float w1 = a1_w[row * s2 + a];
            if (!(w1 > 0.0f)) continue;                      /* R3: inactive slot */
            const int32_t j = a1_idx[row * s2 + a];
            if (j < 0 || j >= n) { ++bad; continue; }        /* R8 */
            const int64_t row_j = ((int64_t)b * n + j) * k + h;   /* R1: same channel h */
            for (int e = 0; e < s3; ++e) {
                const float w2 = a2_w[row_j * s3 + e];
                if (!(w2 > 0.0f)) continue;                  /* R3 */
                const int32_t t = a2_idx[row_j * s3 + e];
                if (t < 0 || t >= n) { ++bad; continue; }    /* R8 */
                const float u = w1 * w2;                     /* R2: one fp32 rounding */
                if (u == 0.0f) continue;                     /* R3: underflowed product */
                cand_t[nc] = t;
                cand_u[nc] = u;
                ++nc;
            }
        }

        /* 2. merge duplicates: W_t = sum of u_c over c with t_c = t, ascending c (R2) */
        int32_t ut[ORACLE_MAX_CAND];
        float uw[ORACLE_MAX_CAND];
        int nu = 0;
        for (int c = 0; c < nc; ++c) {
            int m = 0;
            while (m < nu && ut[m] != cand_t[c]) ++m;
            if (m == nu) {
                ut[nu] = cand_t[c];
                uw[nu] = cand_u[c];
                ++nu;
            } else {
                uw[m] = uw[m] + cand_u[c];
            }
        }

        /* 3. order by weight descending, then index ascending (R4); insertion sort */
        for (int x = 1; x < nu; ++x) {
            const int32_t tt = ut[x];
            const float ww = uw[x];
            int y = x - 1;
            while (y >= 0 && (uw[y] < ww || (uw[y] == ww && ut[y] > tt))) {
                ut[y + 1] = ut[y];
                uw[y + 1] = uw[y];
                --y;
            }
            ut[y + 1] = tt;
            uw[y + 1] = ww;
        }

        /* 4. keep the first s1, pad with (0, 0.0f) (R4, R5: no renormalisation) */
        for (int r = 0; r < s1; ++r) {
            out_idx[row * s1 + r] = r < nu ? ut[r] : 0;
            out_w[row * s1 + r] = r < nu ? uw[r] : 0.0f;
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------
 * SER backward   [MPE2]; readings R1-R5, R8, R9.
 *
 * gout [B, n, k, s1]: gradient with respect to the kept weights A'.w (or, if grad_is_log, with
 * respect to ln A'.w, converted here as g / W). For each row the forward's candidates, merge
 * and selection are recomputed exactly as in oracle_ser; then for every candidate
 * c = (a, e) whose target t_c was kept in slot r (W_r > 0):
 *     dw1[b,i,h,a]  += g_r * w2[b,j,h,e]          (j = A1.idx[b,i,h,a])
 *     dw2[b,j,h,e]  += g_r * w1[b,i,h,a]          (summed over every row that reaches it)
 * in fp64. Work is split over (b, h) planes: a row only reaches second-leg rows of its own
 * sequence and channel, so each plane owns its dw1 and dw2 entries.
 * ---------------------------------------------------------------------------------------- */
int64_t oracle_ser_backward(const int32_t *a1_idx, const float *a1_w, int s2,
                            const int32_t *a2_idx, const float *a2_w, int s3,
                            const float *gout, int s1, int grad_is_log,
                            int B, int n, int k, double *dw1, double *dw2)
{
    int64_t bad = 0;
    if (s2 * s3 > ORACLE_MAX_CAND) return -1;

#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
    for (int64_t plane = 0; plane < (int64_t)B * k; ++plane) {
        const int64_t b = plane / k;
        const int h = (int)(plane % k);
        for (int i = 0; i < n; ++i) {
            const int64_t row = ((int64_t)b * n + i) * k + h;
            for (int a = 0; a < s2; ++a) dw1[row * s2 + a] = 0.0;
            for (int e = 0; e < s3; ++e) dw2[row * s3 + e] = 0.0;
        }
        for (int i = 0; i < n; ++i) {
            const int64_t row = ((int64_t)b * n + i) * k + h;
            /* forward, exactly as oracle_ser */
            int32_t cand_t[ORACLE_MAX_CAND], cand_a[ORACLE_MAX_CAND];
            float cand_u[ORACLE_MAX_CAND];
            int64_t cand_r2[ORACLE_MAX_CAND];
            int nc = 0;
            for (int a = 0; a < s2; ++a) {
                const float w1 = a1_w[row * s2 + a];
                if (!(w1 > 0.0f)) continue;
                const int32_t j = a1_idx[row * s2 + a];
                if (j < 0 || j >= n) { ++bad; continue; }
                const int64_t row_j = ((int64_t)b * n + j) * k + h;
                for (int e = 0; e < s3; ++e) {
                    const float w2 = a2_w[row_j * s3 + e];
                    if (!(w2 > 0.0f)) continue;
                    const int32_t t = a2_idx[row_j * s3 + e];
                    if (t < 0 || t >= n) { ++bad; continue; }
                    const float u = w1 * w2;
                    if (u == 0.0f) continue;
                    cand_t[nc] = t;
                    cand_u[nc] = u;
                    cand_a[nc] = a;
                    cand_r2[nc] = row_j * s3 + e;
                    ++nc;
                }
            }
            int32_t ut[ORACLE_MAX_CAND];
            float uw[ORACLE_MAX_CAND];
            int nu = 0;
            for (int c = 0; c < nc; ++c) {
                int m = 0;
                while (m < nu && ut[m] != cand_t[c]) ++m;
                if (m == nu) {
                    ut[nu] = cand_t[c];
                    uw[nu] = cand_u[c];
                    ++nu;
                } else {
                    uw[m] = uw[m] + cand_u[c];
                }
            }
            for (int x = 1; x < nu; ++x) {
                const int32_t tt = ut[x];
                const float ww = uw[x];
                int y = x - 1;
                while (y >= 0 && (uw[y] < ww || (uw[y] == ww && ut[y] > tt))) {
                    ut[y + 1] = ut[y];
                    uw[y + 1] = uw[y];
                    --y;
                }
                ut[y + 1] = tt;
                uw[y + 1] = ww;
            }
            /* backward through the kept merged weights */
            const int kept = nu < s1 ? nu : s1;
            for (int r = 0; r < kept; ++r) {
                double g = (double)gout[row * s1 + r];
                if (grad_is_log) g /= (double)uw[r];
                for (int c = 0; c < nc; ++c) {
                    if (cand_t[c] != ut[r]) continue;
                    const int a = cand_a[c];
                    dw1[row * s2 + a] += g * (double)a2_w[cand_r2[c]];
                    dw2[cand_r2[c]] += g * (double)a1_w[row * s2 + a];
                }
            }
        }
    }
    return bad;
}

/* Scores of the active slots of one (b, i, hq) row (R6-R8). Returns the number of active
 * slots; fills z[], t[] and slot[] (position of each active slot in the edge row). */
static int sea_row_scores(const float *qrow, const float *kk, const int32_t *idx_row,
                          const float *w_row, int s, int64_t b, int n, int hkv, int h, int d,
                          double scale, double *z, int32_t *t, int *slot, int64_t *bad)
{
    int na = 0;
    for (int j = 0; j < s; ++j) {
        const float w = w_row[j];
        if (!(w > 0.0f)) continue;
        const int32_t tj = idx_row[j];
        if (tj < 0 || tj >= n) { ++*bad; continue; }
        const float *krow = kk + (((int64_t)b * n + tj) * hkv + h) * d;
        double dot = 0.0;
        for (int x = 0; x < d; ++x) dot += (double)qrow[x] * (double)krow[x];
        z[na] = scale * dot + log((double)w);
        t[na] = tj;
        slot[na] = j;
        ++na;
    }
    return na;
}

/* ------------------------------------------------------------------------------------------
 * SEA forward   [KC3], [MPE3]; readings R6-R8.
 *
 * rows: optional list of flat positions b*n + i to evaluate (NULL: all B*n, in order);
 * o [nrows, hq, d] and lse [nrows, hq] are compact over that list.
 * ---------------------------------------------------------------------------------------- */
int64_t oracle_sea_forward(const float *q, const float *kk, const float *vv,
                           const int32_t *idx, const float *w, int s,
                           int B, int n, int hq, int hkv, int d, double scale,
                           const int64_t *rows, int64_t nrows, double *o, double *lse)
{
    const int G = hq / hkv;
    if (rows == NULL) nrows = (int64_t)B * n;
    int64_t bad = 0;

#pragma omp parallel for schedule(static) reduction(+ : bad)
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t bi = rows ? rows[r] : r;
        const int64_t b = bi / n;
        double *z = (double *)malloc(sizeof(double) * (size_t)s);
        int32_t *t = (int32_t *)malloc(sizeof(int32_t) * (size_t)s);
        int *slot = (int *)malloc(sizeof(int) * (size_t)s);
        for (int hqi = 0; hqi < hq; ++hqi) {
            const int h = hqi / G;                                   /* R7 */
            const float *qrow = q + (bi * hq + hqi) * d;
            const int32_t *idx_row = idx + (bi * hkv + h) * s;
            const float *w_row = w + (bi * hkv + h) * s;
            double *orow = o + (r * hq + hqi) * d;
            const int na = sea_row_scores(qrow, kk, idx_row, w_row, s, b, n, hkv, h, d, scale,
                                          z, t, slot, &bad);
            for (int x = 0; x < d; ++x) orow[x] = 0.0;
            if (na == 0) {
                lse[r * hq + hqi] = -INFINITY;
                continue;
            }
            double m = z[0];
            for (int a = 1; a < na; ++a) m = z[a] > m ? z[a] : m;
            double l = 0.0;
            for (int a = 0; a < na; ++a) l += exp(z[a] - m);
            for (int a = 0; a < na; ++a) {
                const double p = exp(z[a] - m) / l;
                const float *vrow = vv + (((int64_t)b * n + t[a]) * hkv + h) * d;
                for (int x = 0; x < d; ++x) orow[x] += p * (double)vrow[x];
            }
            lse[r * hq + hqi] = m + log(l);
        }
        free(z);
        free(t);
        free(slot);
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------
 * SEA backward (fp64): gradients of the SEA forward above with respect to q, K, V and
 * ln w, given the upstream gradient dO of o. Indices get none [MPE2].
 *
 *   p_j  = softmax_j(z)                  (recomputed from the forward definition)
 *   D    = <dO, o>
 *   dz_j = p_j * (<dO, V[t_j]> - D)
 *   dq           = scale * sum_j dz_j K[t_j]
 *   dK[t_j]     += scale * dz_j q
 *   dV[t_j]     += p_j dO
 *   dlogw[.., j] += dz_j                 (summed over the query heads of the KV head)
 * Inactive slots get 0. Work is split over (b, h) planes, each of which owns its dK/dV
 * rows, dlogw rows and the dq rows of its query heads, so every sum runs serially in a fixed
 * order.
 * ---------------------------------------------------------------------------------------- */
int64_t oracle_sea_backward(const float *q, const float *kk, const float *vv, const float *dout,
                            const int32_t *idx, const float *w, int s,
                            int B, int n, int hq, int hkv, int d, double scale,
                            double *dq, double *dk, double *dv, double *dlogw)
{
    const int G = hq / hkv;
    int64_t bad = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
    for (int64_t plane = 0; plane < (int64_t)B * hkv; ++plane) {
        const int64_t b = plane / hkv;
        const int h = (int)(plane % hkv);
        double *z = (double *)malloc(sizeof(double) * (size_t)s);
        int32_t *t = (int32_t *)malloc(sizeof(int32_t) * (size_t)s);
        int *slot = (int *)malloc(sizeof(int) * (size_t)s);
        double *orow = (double *)malloc(sizeof(double) * (size_t)d);

        for (int i = 0; i < n; ++i) {
            const int64_t kvrow = ((int64_t)b * n + i) * hkv + h;
            for (int x = 0; x < d; ++x) dk[kvrow * d + x] = 0.0;
            for (int x = 0; x < d; ++x) dv[kvrow * d + x] = 0.0;
        }
        for (int i = 0; i < n; ++i) {
            const int64_t bi = (int64_t)b * n + i;
            const int32_t *idx_row = idx + (bi * hkv + h) * s;
            const float *w_row = w + (bi * hkv + h) * s;
            double *glw = dlogw + (bi * hkv + h) * s;
            for (int j = 0; j < s; ++j) glw[j] = 0.0;

            for (int hqi = h * G; hqi < (h + 1) * G; ++hqi) {
                const float *qrow = q + (bi * hq + hqi) * d;
                const float *grow = dout + (bi * hq + hqi) * d;
                double *dqrow = dq + (bi * hq + hqi) * d;
                for (int x = 0; x < d; ++x) dqrow[x] = 0.0;
                const int na = sea_row_scores(qrow, kk, idx_row, w_row, s, b, n, hkv, h, d,
                                              scale, z, t, slot, &bad);
                if (na == 0) continue;

                /* forward: p and o */
                double m = z[0];
                for (int a = 1; a < na; ++a) m = z[a] > m ? z[a] : m;
                double l = 0.0;
                for (int a = 0; a < na; ++a) l += exp(z[a] - m);
                for (int x = 0; x < d; ++x) orow[x] = 0.0;
                for (int a = 0; a < na; ++a) {
                    const double p = exp(z[a] - m) / l;
                    const float *vrow = vv + (((int64_t)b * n + t[a]) * hkv + h) * d;
                    for (int x = 0; x < d; ++x) orow[x] += p * (double)vrow[x];
                }
                double D = 0.0;
                for (int x = 0; x < d; ++x) D += (double)grow[x] * orow[x];

                /* backward through softmax, the scores and the weighted sum */
                for (int a = 0; a < na; ++a) {
                    const double p = exp(z[a] - m) / l;
                    const int64_t tr = ((int64_t)b * n + t[a]) * hkv + h;
                    const float *krow = kk + tr * d;
                    const float *vrow = vv + tr * d;
                    double dp = 0.0;
                    for (int x = 0; x < d; ++x) dp += (double)grow[x] * (double)vrow[x];
                    const double dz = p * (dp - D);
                    for (int x = 0; x < d; ++x) dqrow[x] += scale * dz * (double)krow[x];
                    for (int x = 0; x < d; ++x) dk[tr * d + x] += scale * dz * (double)qrow[x];
                    for (int x = 0; x < d; ++x) dv[tr * d + x] += p * (double)grow[x];
                    glw[slot[a]] += dz;
                }
            }
        }
        free(z);
        free(t);
        free(slot);
        free(orow);
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------
 * Leg sparsification   [MPE2] (the stored edges are mixed into a pair of legs and each leg is
 * sparsified before the composition), [MF4]; readings R3, R4, R5, R8, R10, R11.
 *
 * Shared by the forward and the backward below: merge the candidates of one row by target
 * (ascending candidate order, fp32 adds) and order the distinct targets by weight descending,
 * then target ascending. Returns the number of distinct targets.
 * ---------------------------------------------------------------------------------------- */
static int merge_and_order(const int32_t *cand_t, const float *cand_u, int nc,
                           int32_t *ut, float *uw)
{
    int nu = 0;
    for (int c = 0; c < nc; ++c) {
        int m = 0;
        while (m < nu && ut[m] != cand_t[c]) ++m;
        if (m == nu) {
            ut[nu] = cand_t[c];
            uw[nu] = cand_u[c];
            ++nu;
        } else {
            uw[m] = uw[m] + cand_u[c];
        }
    }
    for (int x = 1; x < nu; ++x) {
        const int32_t tt = ut[x];
        const float ww = uw[x];
        int y = x - 1;
        while (y >= 0 && (uw[y] < ww || (uw[y] == ww && ut[y] > tt))) {
            ut[y + 1] = ut[y];
            uw[y + 1] = uw[y];
            --y;
        }
        ut[y + 1] = tt;
        uw[y + 1] = ww;
    }
    return nu;
}

/* Candidates of leg channel h at one token (R10). valid[c*s0+a] says whether stored edge (c, a)
 * is active and in range; cand_ca receives each candidate's c*s0 + a. Returns their number. */
static int leg_candidates(const int32_t *e_idx_tok, const float *e_w_tok, const uint8_t *valid,
                          const float *mix_tok, int h, int k, int s0,
                          int32_t *cand_t, float *cand_u, int *cand_ca)
{
    int nc = 0;
    for (int c = 0; c < k; ++c) {
        const float m = mix_tok[h * k + c];
        for (int a = 0; a < s0; ++a) {
            const int ca = c * s0 + a;
            if (!valid[ca]) continue;
            const float u = m * e_w_tok[ca];          /* one fp32 rounding, as R2 */
            if (u == 0.0f) continue;                   /* R3 */
            cand_t[nc] = e_idx_tok[ca];
            cand_u[nc] = u;
            cand_ca[nc] = ca;
            ++nc;
        }
    }
    return nc;
}

/* Active, in-range stored edges of one token (R3, R8); returns how many active ones were out
 * of range. */
static int64_t leg_valid(const int32_t *e_idx_tok, const float *e_w_tok, int ks0, int n,
                         uint8_t *valid)
{
    int64_t bad = 0;
    for (int ca = 0; ca < ks0; ++ca) {
        valid[ca] = 0;
        if (!(e_w_tok[ca] > 0.0f)) continue;
        if (e_idx_tok[ca] < 0 || e_idx_tok[ca] >= n) { ++bad; continue; }
        valid[ca] = 1;
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------
 * Forward: for every (b, i, h), A1[b,i,h,:] = Sparsify_s2(mix of token i's stored edges by
 * M1[b,i,h,:]) and A2[b,i,h,:] = Sparsify_s3(the same with M2). E is [B, n, k, s0]; M1 and M2
 * are [B, n, k, k] read at token offset (b*n + i) * mix_tok_stride (k*k, or 0 for one shared
 * [k, k] matrix). Returns the number of active stored edges out of range (each counted once).
 * ---------------------------------------------------------------------------------------- */
int64_t oracle_leg_sparsify(const int32_t *e_idx, const float *e_w, int s0, int k,
                            const float *mix1, const float *mix2, int64_t mix_tok_stride,
                            int32_t *a1_idx, float *a1_w, int s2,
                            int32_t *a2_idx, float *a2_w, int s3, int B, int n)
{
    const int ks0 = k * s0;
    int64_t bad = 0;
    if (ks0 > ORACLE_MAX_CAND) return -1;

#pragma omp parallel for schedule(static) reduction(+ : bad)
    for (int64_t tok = 0; tok < (int64_t)B * n; ++tok) {
        const int32_t *ei = e_idx + tok * ks0;
        const float *ew = e_w + tok * ks0;
        uint8_t valid[ORACLE_MAX_CAND];
        bad += leg_valid(ei, ew, ks0, n, valid);
        for (int leg = 0; leg < 2; ++leg) {
            const float *mix = (leg == 0 ? mix1 : mix2) + tok * mix_tok_stride;
            const int sl = leg == 0 ? s2 : s3;
            int32_t *oi = leg == 0 ? a1_idx : a2_idx;
            float *ow = leg == 0 ? a1_w : a2_w;
            for (int h = 0; h < k; ++h) {
                int32_t cand_t[ORACLE_MAX_CAND], ut[ORACLE_MAX_CAND];
                float cand_u[ORACLE_MAX_CAND], uw[ORACLE_MAX_CAND];
                int cand_ca[ORACLE_MAX_CAND];
                const int nc = leg_candidates(ei, ew, valid, mix, h, k, s0, cand_t, cand_u, cand_ca);
                const int nu = merge_and_order(cand_t, cand_u, nc, ut, uw);
                const int64_t row = tok * k + h;
                for (int r = 0; r < sl; ++r) {           /* R4 padding, R5 */
                    oi[row * sl + r] = r < nu ? ut[r] : 0;
                    ow[row * sl + r] = r < nu ? uw[r] : 0.0f;
                }
            }
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------
 * Backward of the leg sparsification   [MPE2]; readings R10-R12.
 *
 * g1 [B, n, k, s2] and g2 [B, n, k, s3]: gradients with respect to the kept leg weights. The
 * forward's candidates, merge and selection are recomputed; then for every candidate (c, a)
 * merged into a kept slot r (W_r > 0) of leg L, channel h:
 *     dew[b,i,c,a]      += g_L[b,i,h,r] * M_L[b,i,h,c]
 *     dmix_L[b,i,h,c]   += g_L[b,i,h,r] * E.w[b,i,c,a]
 * in fp64, over every active stored edge (c, a) reaching t_r, including those whose product
 * was zero (R12). Each token owns its outputs, so tokens run in parallel.
 * ---------------------------------------------------------------------------------------- */
int64_t oracle_leg_backward(const int32_t *e_idx, const float *e_w, int s0, int k,
                            const float *mix1, const float *mix2, int64_t mix_tok_stride,
                            const float *g1, int s2, const float *g2, int s3, int B, int n,
                            double *dew, double *dmix1, double *dmix2)
{
    const int ks0 = k * s0;
    int64_t bad = 0;
    if (ks0 > ORACLE_MAX_CAND) return -1;

#pragma omp parallel for schedule(static) reduction(+ : bad)
    for (int64_t tok = 0; tok < (int64_t)B * n; ++tok) {
        const int32_t *ei = e_idx + tok * ks0;
        const float *ew = e_w + tok * ks0;
        uint8_t valid[ORACLE_MAX_CAND];
        bad += leg_valid(ei, ew, ks0, n, valid);
        for (int ca = 0; ca < ks0; ++ca) dew[tok * ks0 + ca] = 0.0;
        for (int x = 0; x < k * k; ++x) {
            dmix1[tok * k * k + x] = 0.0;
            dmix2[tok * k * k + x] = 0.0;
        }
        for (int leg = 0; leg < 2; ++leg) {
            const float *mix = (leg == 0 ? mix1 : mix2) + tok * mix_tok_stride;
            const int sl = leg == 0 ? s2 : s3;
            const float *g = leg == 0 ? g1 : g2;
            double *dmix = (leg == 0 ? dmix1 : dmix2) + tok * k * k;
            for (int h = 0; h < k; ++h) {
                int32_t cand_t[ORACLE_MAX_CAND], ut[ORACLE_MAX_CAND];
                float cand_u[ORACLE_MAX_CAND], uw[ORACLE_MAX_CAND];
                int cand_ca[ORACLE_MAX_CAND];
                const int nc = leg_candidates(ei, ew, valid, mix, h, k, s0, cand_t, cand_u, cand_ca);
                const int nu = merge_and_order(cand_t, cand_u, nc, ut, uw);
                const int kept = nu < sl ? nu : sl;
                const int64_t row = tok * k + h;
                /* every active stored edge whose target was kept carries the derivative,
                 * also one whose product with its coefficient was zero (R12) */
                for (int r = 0; r < kept; ++r) {
                    const double gr = (double)g[row * sl + r];
                    for (int ca = 0; ca < ks0; ++ca) {
                        if (!valid[ca] || ei[ca] != ut[r]) continue;
                        const int c = ca / s0;
                        dew[tok * ks0 + ca] += gr * (double)mix[h * k + c];
                        dmix[h * k + c] += gr * (double)ew[ca];
                    }
                }
            }
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------
 * SER with refresh edges: A' = Sparsify_s1(A1 A2 + F)   [MPE2], [MF5]; readings R1-R5, R8, R13.
 *
 * Candidates of row (b, i, h): the s2*s3 two-hop paths exactly as oracle_ser forms them, then
 * the sf refresh slots f_idx/f_w[b,i,h,f] (weight > 0, index in range) with their own weights.
 * cand_src[x] records where candidate x came from: the path slot pair (a, e) as a*s3 + e with
 * its second-leg row, or a refresh slot as -(f + 1).
 * ---------------------------------------------------------------------------------------- */
static int ser_refresh_candidates(const int32_t *a1_idx, const float *a1_w, int s2,
                                  const int32_t *a2_idx, const float *a2_w, int s3,
                                  const int32_t *f_idx, const float *f_w, int sf,
                                  int64_t row, int64_t b, int h, int n, int k,
                                  int32_t *cand_t, float *cand_u, int *cand_src,
                                  int64_t *cand_r2, int64_t *bad)
{
    int nc = 0;
    for (int a = 0; a < s2; ++a) {
        const float w1 = a1_w[row * s2 + a];
        if (!(w1 > 0.0f)) continue;
        const int32_t j = a1_idx[row * s2 + a];
        if (j < 0 || j >= n) { ++*bad; continue; }
        const int64_t row_j = ((int64_t)b * n + j) * k + h;
        for (int e = 0; e < s3; ++e) {
            const float w2 = a2_w[row_j * s3 + e];
            if (!(w2 > 0.0f)) continue;
            const int32_t t = a2_idx[row_j * s3 + e];
            if (t < 0 || t >= n) { ++*bad; continue; }
            const float u = w1 * w2;
            if (u == 0.0f) continue;
            cand_t[nc] = t;
            cand_u[nc] = u;
            cand_src[nc] = a * s3 + e;
            cand_r2[nc] = row_j * s3 + e;
            ++nc;
        }
    }
    for (int f = 0; f < sf; ++f) {
        const float w = f_w[row * sf + f];
        if (!(w > 0.0f)) continue;
        const int32_t t = f_idx[row * sf + f];
        if (t < 0 || t >= n) { ++*bad; continue; }
        cand_t[nc] = t;
        cand_u[nc] = w;
        cand_src[nc] = -(f + 1);
        cand_r2[nc] = -1;
        ++nc;
    }
    return nc;
}

int64_t oracle_ser_refresh(const int32_t *a1_idx, const float *a1_w, int s2,
                           const int32_t *a2_idx, const float *a2_w, int s3,
                           const int32_t *f_idx, const float *f_w, int sf,
                           int32_t *out_idx, float *out_w, int s1, int B, int n, int k)
{
    const int64_t rows = (int64_t)B * n * k;
    int64_t bad = 0;
    if (s2 * s3 + sf > ORACLE_MAX_CAND) return -1;

#pragma omp parallel for schedule(static) reduction(+ : bad)
    for (int64_t row = 0; row < rows; ++row) {
        const int h = (int)(row % k);
        const int64_t b = row / ((int64_t)n * k);
        int32_t cand_t[ORACLE_MAX_CAND], ut[ORACLE_MAX_CAND];
        float cand_u[ORACLE_MAX_CAND], uw[ORACLE_MAX_CAND];
        int cand_src[ORACLE_MAX_CAND];
        int64_t cand_r2[ORACLE_MAX_CAND];
        int64_t my_bad = 0;
        const int nc = ser_refresh_candidates(a1_idx, a1_w, s2, a2_idx, a2_w, s3, f_idx, f_w, sf,
                                              row, b, h, n, k, cand_t, cand_u, cand_src, cand_r2,
                                              &my_bad);
        bad += my_bad;
        const int nu = merge_and_order(cand_t, cand_u, nc, ut, uw);
        for (int r = 0; r < s1; ++r) {
            out_idx[row * s1 + r] = r < nu ? ut[r] : 0;
            out_w[row * s1 + r] = r < nu ? uw[r] : 0.0f;
        }
    }
    return bad;
}

/* Backward of oracle_ser_refresh (R9, R13): for every candidate merged into a kept slot r,
 *     a path (a, e):    dw1[b,i,h,a] += g_r * w2,  dw2[b,j,h,e] += g_r * w1
 *     a refresh slot f: dfw[b,i,h,f] += g_r
 * in fp64; g_r as oracle_ser_backward (divided by W_r when grad_is_log). */
int64_t oracle_ser_refresh_backward(const int32_t *a1_idx, const float *a1_w, int s2,
                                    const int32_t *a2_idx, const float *a2_w, int s3,
                                    const int32_t *f_idx, const float *f_w, int sf,
                                    const float *gout, int s1, int grad_is_log,
                                    int B, int n, int k, double *dw1, double *dw2, double *dfw)
{
    int64_t bad = 0;
    if (s2 * s3 + sf > ORACLE_MAX_CAND) return -1;

#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
    for (int64_t plane = 0; plane < (int64_t)B * k; ++plane) {
        const int64_t b = plane / k;
        const int h = (int)(plane % k);
        for (int i = 0; i < n; ++i) {
            const int64_t row = ((int64_t)b * n + i) * k + h;
            for (int a = 0; a < s2; ++a) dw1[row * s2 + a] = 0.0;
            for (int e = 0; e < s3; ++e) dw2[row * s3 + e] = 0.0;
            for (int f = 0; f < sf; ++f) dfw[row * sf + f] = 0.0;
        }
        for (int i = 0; i < n; ++i) {
            const int64_t row = ((int64_t)b * n + i) * k + h;
            int32_t cand_t[ORACLE_MAX_CAND], ut[ORACLE_MAX_CAND];
            float cand_u[ORACLE_MAX_CAND], uw[ORACLE_MAX_CAND];
            int cand_src[ORACLE_MAX_CAND];
            int64_t cand_r2[ORACLE_MAX_CAND];
            int64_t my_bad = 0;
            const int nc = ser_refresh_candidates(a1_idx, a1_w, s2, a2_idx, a2_w, s3, f_idx, f_w,
                                                  sf, row, b, h, n, k, cand_t, cand_u, cand_src,
                                                  cand_r2, &my_bad);
            bad += my_bad;
            const int nu = merge_and_order(cand_t, cand_u, nc, ut, uw);
            const int kept = nu < s1 ? nu : s1;
            for (int r = 0; r < kept; ++r) {
                double g = (double)gout[row * s1 + r];
                if (grad_is_log) g /= (double)uw[r];
                for (int x = 0; x < nc; ++x) {
                    if (cand_t[x] != ut[r]) continue;
                    if (cand_src[x] < 0) {
                        dfw[row * sf + (-cand_src[x] - 1)] += g;
                    } else {
                        const int a = cand_src[x] / s3;
                        dw1[row * s2 + a] += g * (double)a2_w[cand_r2[x]];
                        dw2[cand_r2[x]] += g * (double)a1_w[row * s2 + a];
                    }
                }
            }
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------
 * Refresh edges from the latest dense attention layer   [MF5], and the last sentence of the
 * referral paragraph of "Methodology in Plain English": refresh edges are the input edges or
 * the top positions of the most recent dense attention layer. Readings R14, R15.
 * ---------------------------------------------------------------------------------------- */

/* <q[b,i,hq], k[b,t,h]> in fp64 on inputs widened exactly from fp32 / bf16. */
static double dense_dot(const float *q, const float *kk, int64_t b, int i, int t, int hqi, int h,
                        int n, int hq, int hkv, int d)
{
    const float *qrow = q + (((int64_t)b * n + i) * hq + hqi) * d;
    const float *krow = kk + (((int64_t)b * n + t) * hkv + h) * d;
    double dot = 0.0;
    for (int x = 0; x < d; ++x) dot += (double)qrow[x] * (double)krow[x];
    return dot;
}

/* lse [nrows, hq]: log of sum over t <= i of exp(scale <q[b,i,hq], k[b,t,h]>), the normaliser
 * of causal softmax attention (R14), for the flat positions rows[r] = b*n + i (NULL: all B*n
 * in order). */
void oracle_dense_lse(const float *q, const float *kk, int B, int n, int hq, int hkv, int d,
                      double scale, const int64_t *rows, int64_t nrows, double *lse)
{
    const int G = hq / hkv;
    if (rows == NULL) nrows = (int64_t)B * n;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t bi = rows ? rows[r] : r;
        const int64_t b = bi / n;
        const int i = (int)(bi % n);
        double *z = (double *)malloc(sizeof(double) * (size_t)(i + 1));
        for (int hqi = 0; hqi < hq; ++hqi) {
            const int h = hqi / G;
            double m = -INFINITY;
            for (int t = 0; t <= i; ++t) {
                z[t] = scale * dense_dot(q, kk, b, i, t, hqi, h, n, hq, hkv, d);
                m = z[t] > m ? z[t] : m;
            }
            double l = 0.0;
            for (int t = 0; t <= i; ++t) l += exp(z[t] - m);
            lse[r * hq + hqi] = m + log(l);
        }
        free(z);
    }
}

/* Attention mass of KV head h at every position (R14, R15): mass[r, h, t] = mean over the
 * group's query heads of exp(scale <q, k[t]> - lse) for t <= i, 0 for t > i, for the flat
 * positions rows[r] = b*n + i (NULL: all B*n in order). */
void oracle_dense_mass(const float *q, const float *kk, const float *lse, int B, int n, int hq,
                       int hkv, int d, double scale, const int64_t *rows, int64_t nrows,
                       double *mass)
{
    const int G = hq / hkv;
    if (rows == NULL) nrows = (int64_t)B * n;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t bi = rows ? rows[r] : r;
        const int64_t b = bi / n;
        const int i = (int)(bi % n);
        for (int h = 0; h < hkv; ++h) {
            double *mrow = mass + (r * hkv + h) * (int64_t)n;
            for (int t = 0; t < n; ++t) mrow[t] = 0.0;
            for (int hqi = h * G; hqi < (h + 1) * G; ++hqi) {
                const double l = (double)lse[bi * hq + hqi];
                for (int t = 0; t <= i; ++t)
                    mrow[t] += exp(scale * dense_dot(q, kk, b, i, t, hqi, h, n, hq, hkv, d) - l);
            }
            for (int t = 0; t <= i; ++t) mrow[t] /= (double)G;
        }
    }
}

typedef struct {
    double mass;
    int32_t t;
} dense_entry;

/* mass descending, then position ascending (R15) */
static int dense_entry_order(const void *pa, const void *pb)
{
    const dense_entry *a = (const dense_entry *)pa, *b = (const dense_entry *)pb;
    if (a->mass != b->mass) return a->mass > b->mass ? -1 : 1;
    return (a->t > b->t) - (a->t < b->t);
}

/* Refresh edges [nrows, hkv, sf] (R15) from the masses of oracle_dense_mass: all positions
 * t <= i sorted by (mass desc, t asc), the first sf kept, the rest padded with (0, 0.0f). */
void oracle_dense_refresh(const float *q, const float *kk, const float *lse, int B, int n,
                          int hq, int hkv, int d, double scale, int sf, const int64_t *rows,
                          int64_t nrows, int32_t *out_idx, float *out_w)
{
    if (rows == NULL) nrows = (int64_t)B * n;
    double *mass = (double *)malloc(sizeof(double) * (size_t)nrows * hkv * n);
    oracle_dense_mass(q, kk, lse, B, n, hq, hkv, d, scale, rows, nrows, mass);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t bi = rows ? rows[r] : r;
        const int i = (int)(bi % n);
        dense_entry *e = (dense_entry *)malloc(sizeof(dense_entry) * (size_t)(i + 1));
        for (int h = 0; h < hkv; ++h) {
            for (int t = 0; t <= i; ++t) {
                e[t].mass = mass[(r * hkv + h) * (int64_t)n + t];
                e[t].t = t;
            }
            qsort(e, (size_t)(i + 1), sizeof(dense_entry), dense_entry_order);
            for (int f = 0; f < sf; ++f) {
                out_idx[(r * hkv + h) * sf + f] = f <= i ? e[f].t : 0;
                out_w[(r * hkv + h) * sf + f] = f <= i ? (float)e[f].mass : 0.0f;
            }
        }
        free(e);
    }
    free(mass);
}
