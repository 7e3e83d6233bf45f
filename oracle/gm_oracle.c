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
