/*
 * hkv_oracle.c -- plain, slow CPU oracle of one HARD-KV Cascade Cache decode
 * step, written directly from the definitions of the paper pages.
 *
 * TEST INFRASTRUCTURE ONLY: only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg load it. It shares no code with the CUDA
 * library.
 *
 * Citations name the page and its section:
 *   [Abstract]  arXiv abstract of "HARD-KV: Head-Adaptive Regularization for
 *               Decoding-time KV Compression" (mlsanity.com paper page);
 *   [TS 2.A]    gist.science Technical Summary of the same paper, section 2.A
 *               "Cascade Cache Hierarchy"; [TS 2.B] "Logits Calibration
 *               Mechanism"; [TS 2.C] "System-Aware Index Regularization";
 *               [TS 3] "Key Contributions".
 *
 * Arithmetic: every dot product, sum, exponential and logarithm is done in
 * IEEE double, sequentially in index order; a value is rounded to float only
 * where it is stored as a float result. Parallelism is only across units
 * (one KV head of one sequence), whose results are independent.
 */
#include "hkv_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- element access ----------------------------------------------------- */

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_to_double(uint16_t bits)
{
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

static double elem(const void *base, int32_t dtype, int64_t i)
{
    if (dtype == HKVO_BF16)
        return bf16_to_double(((const uint16_t *)base)[i]);
    return (double)((const float *)base)[i];
}

static int64_t row_off(const hkvo_tier *t, int32_t b, int32_t h, int64_t j)
{
    return (int64_t)b * t->sb + (int64_t)h * t->sh + j * t->st;
}

static int tier_len(const hkvo_tier *t, int32_t u)
{
    if (t == NULL || t->len == NULL)
        return 0;
    return t->len[u];
}

static int check_dims(const hkvo_dims *d)
{
    if (d == NULL || d->B < 0 || d->Hq <= 0 || d->Hkv <= 0 || d->D <= 0)
        return -1;
    if (d->Hq % d->Hkv != 0)
        return -1;
    if (d->dtype != HKVO_BF16 && d->dtype != HKVO_F32)
        return -1;
    return 0;
}

static int check_tier(const hkvo_tier *t, int32_t units)
{
    if (t == NULL)
        return 0;
    if (t->len == NULL || t->cap < 0)
        return -1;
    for (int32_t u = 0; u < units; ++u)
        if (t->len[u] < 0 || t->len[u] > t->cap)
            return -1;
    return 0;
}

/* q . K_j for query head hq, in double. */
static double dot_qk(const hkvo_dims *d, const void *q, int32_t b, int32_t hq,
                     const hkvo_tier *t, int32_t h, int64_t j)
{
    int64_t qo = ((int64_t)b * d->Hq + hq) * d->D;
    int64_t ko = row_off(t, b, h, j);
    double s = 0.0;
    for (int32_t x = 0; x < d->D; ++x)
        s += elem(q, d->dtype, qo + x) * elem(t->k, d->dtype, ko + x);
    return s;
}

/* ---- S1: scoring -------------------------------------------------------- */

/* [TS 2.B] names max-pooled logits as the importance metric; the scores are
 * the attention scores of the group's query heads ([TS 2.B] "temperature of
 * the attention scores"). Pooling is over the G query heads that share KV head
 * h; no pooling along the token axis. */
int hkvo_score(const hkvo_dims *d, const void *q, const hkvo_tier *sp, float *z,
               int32_t zcap)
{
    if (check_dims(d) || sp == NULL || z == NULL)
        return -1;
    int32_t units = d->B * d->Hkv;
    if (check_tier(sp, units) || zcap < sp->cap)
        return -1;
    int32_t G = d->Hq / d->Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t u = 0; u < units; ++u) {
        int32_t b = u / d->Hkv, h = u % d->Hkv;
        for (int32_t j = 0; j < sp->len[u]; ++j) {
            double best = -INFINITY;
            for (int32_t g = 0; g < G; ++g) {
                double s = d->scale * dot_qk(d, q, b, h * G + g, sp, h, j);
                if (s > best)
                    best = s;
            }
            z[(int64_t)u * zcap + j] = (float)best;
        }
    }
    return 0;
}

/* ---- S2: Logits Calibration -------------------------------------------- */

/* [TS 2.B]: importance values are mapped to a normalised softmax by adjusting
 * the temperature of the scores; [TS 3]: onto the raw attention distribution.
 * Reading: P_j = exp(beta (z_j - m)) / Z over the sparse tier, beta given per
 * unit (1 = the raw distribution of the max-pooled logits). */
static double calib_weight(float zj, float m, double beta)
{
    if (zj == m || beta == 0.0)
        return 1.0;
    return exp(beta * ((double)zj - (double)m));
}

static int unit_max(const float *zu, int32_t n, float *m)
{
    float best = -INFINITY;
    for (int32_t j = 0; j < n; ++j) {
        if (zu[j] != zu[j])
            return -2; /* NaN score: undefined, refused */
        if (zu[j] > best)
            best = zu[j];
    }
    *m = best;
    return 0;
}

int hkvo_calibrate(int32_t units, const float *z, int32_t zcap, const int32_t *len,
                   const float *beta, float *P, float *m, float *logZ)
{
    if (z == NULL || len == NULL || units < 0)
        return -1;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : err)
    for (int32_t u = 0; u < units; ++u) {
        const float *zu = z + (int64_t)u * zcap;
        int32_t n = len[u];
        double bu = beta ? (double)beta[u] : 1.0;
        float mu;
        if (unit_max(zu, n, &mu)) {
            err = -2;
            continue;
        }
        double Z = 0.0;
        for (int32_t j = 0; j < n; ++j)
            Z += calib_weight(zu[j], mu, bu);
        if (P)
            for (int32_t j = 0; j < n; ++j)
                P[(int64_t)u * zcap + j] = (float)(calib_weight(zu[j], mu, bu) / Z);
        if (m)
            m[u] = mu;
        if (logZ)
            logZ[u] = n > 0 ? (float)log(Z) : -INFINITY;
    }
    return err;
}

/* ---- S3: Top-p budget ---------------------------------------------------- */

/* Order of the sparse tokens: score descending, then lower token index first.
 * Float comparison treats -0 and +0 as equal. */
typedef struct {
    float z;
    int32_t j;
} scored;

static int by_score_desc(const void *a, const void *b)
{
    const scored *x = (const scored *)a, *y = (const scored *)b;
    if (x->z > y->z)
        return -1;
    if (x->z < y->z)
        return 1;
    return (x->j > y->j) - (x->j < y->j);
}

static scored *sorted_unit(const float *zu, int32_t n)
{
    scored *s = (scored *)malloc(sizeof(scored) * (size_t)(n > 0 ? n : 1));
    if (s == NULL)
        return NULL;
    for (int32_t j = 0; j < n; ++j) {
        s[j].z = zu[j];
        s[j].j = j;
    }
    qsort(s, (size_t)n, sizeof(scored), by_score_desc);
    return s;
}

/* [Abstract], [TS 2.A]: per-head Top-p (nucleus) budget -- the fewest tokens,
 * taken in descending calibrated probability, whose mass is at least p --
 * clamped to the hard limits [bmin, bmax] and to the tokens present. */
static void topp_unit(const float *zu, int32_t n, double beta, float p,
                      int32_t bmin, int32_t bmax, int32_t *k_out, int32_t *kstar_out,
                      double *cb_out, double *ca_out, int *err)
{
    int32_t kstar = 0;
    double c_before = 0.0, c_at = 0.0;
    float mu;
    if (unit_max(zu, n, &mu)) {
        *err = -2;
        return;
    }
    if (n == 0) {
        kstar = 0;
    } else if (p >= 1.0f) {
        kstar = n;
    } else if (p <= 0.0f) {
        kstar = 0;
    } else {
        scored *s = sorted_unit(zu, n);
        if (s == NULL) {
            *err = -3;
            return;
        }
        double Z = 0.0;
        for (int32_t j = 0; j < n; ++j)
            Z += calib_weight(zu[j], mu, beta);
        double C = 0.0;
        kstar = n;
        for (int32_t i = 0; i < n; ++i) {
            double Pi = calib_weight(s[i].z, mu, beta) / Z;
            c_before = C;
            C += Pi;
            if (C >= (double)p) {
                kstar = i + 1;
                break;
            }
        }
        c_at = C;
        free(s);
    }
    int32_t k = kstar < bmax ? kstar : bmax;
    if (k < bmin)
        k = bmin;
    if (k > n)
        k = n;
    *k_out = k;
    if (kstar_out)
        *kstar_out = kstar;
    if (cb_out)
        *cb_out = c_before;
    if (ca_out)
        *ca_out = c_at;
}

int hkvo_topp(int32_t units, const float *z, int32_t zcap, const int32_t *len,
              const float *beta, float p, const float *p_unit, int32_t bmin,
              int32_t bmax, int32_t *k, int32_t *kstar, double *c_before,
              double *c_at)
{
    if (z == NULL || len == NULL || k == NULL || bmin < 0 || bmin > bmax)
        return -1;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : err)
    for (int32_t u = 0; u < units; ++u) {
        int e = 0;
        topp_unit(z + (int64_t)u * zcap, len[u], beta ? (double)beta[u] : 1.0,
                  p_unit ? p_unit[u] : p, bmin, bmax, &k[u], kstar ? &kstar[u] : NULL,
                  c_before ? &c_before[u] : NULL, c_at ? &c_at[u] : NULL, &e);
        if (e < err)
            err = e;
    }
    return err;
}

/* ---- S4: Index Regularization -------------------------------------------- */

static int by_index(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* [TS 2.C] Flatten Index: the selected indices regularised to the maximum
 * length (PAD_MAX) or to the sum of lengths (FLAT_SUM); each row keeps the
 * tokens in their original order (ascending index). */
int hkvo_compact(int32_t units, const float *z, int32_t zcap, const int32_t *len,
                 const int32_t *sel_len, int32_t bmax, int32_t layout, int32_t *idx,
                 int32_t *offsets)
{
    if (z == NULL || len == NULL || sel_len == NULL || idx == NULL || bmax < 0)
        return -1;
    if (layout != HKVO_PAD_MAX && layout != HKVO_FLAT_SUM)
        return -1;
    if (layout == HKVO_FLAT_SUM && offsets == NULL)
        return -1;
    for (int32_t u = 0; u < units; ++u)
        if (sel_len[u] < 0 || sel_len[u] > len[u] || sel_len[u] > bmax)
            return -1;
    if (layout == HKVO_FLAT_SUM) {
        offsets[0] = 0;
        for (int32_t u = 0; u < units; ++u)
            offsets[u + 1] = offsets[u] + sel_len[u];
    }
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : err)
    for (int32_t u = 0; u < units; ++u) {
        int32_t n = len[u], k = sel_len[u];
        int32_t *row = layout == HKVO_PAD_MAX ? idx + (int64_t)u * bmax : idx + offsets[u];
        scored *s = sorted_unit(z + (int64_t)u * zcap, n);
        if (s == NULL) {
            err = -3;
            continue;
        }
        for (int32_t i = 0; i < k; ++i)
            row[i] = s[i].j;
        free(s);
        qsort(row, (size_t)k, sizeof(int32_t), by_index);
        if (layout == HKVO_PAD_MAX)
            for (int32_t i = k; i < bmax; ++i)
                row[i] = -1;
    }
    return err;
}

/* [TS 2.C] Rewrite Cache: the selected rows moved to a contiguous range. */
int hkvo_gather(const hkvo_dims *d, const hkvo_tier *sp, const int32_t *idx,
                const int32_t *sel_len, int32_t bmax, void *kc, void *vc)
{
    if (check_dims(d) || sp == NULL || idx == NULL || sel_len == NULL)
        return -1;
    int32_t units = d->B * d->Hkv;
    size_t es = d->dtype == HKVO_BF16 ? 2 : 4;
    for (int32_t u = 0; u < units; ++u) {
        int32_t b = u / d->Hkv, h = u % d->Hkv;
        for (int32_t i = 0; i < sel_len[u]; ++i) {
            int32_t j = idx[(int64_t)u * bmax + i];
            if (j < 0 || j >= sp->len[u])
                return -1;
            int64_t src = row_off(sp, b, h, j) * (int64_t)es;
            int64_t dst = (((int64_t)u * bmax) + i) * d->D * (int64_t)es;
            if (kc)
                memcpy((char *)kc + dst, (const char *)sp->k + src, (size_t)d->D * es);
            if (vc)
                memcpy((char *)vc + dst, (const char *)sp->v + src, (size_t)d->D * es);
        }
    }
    return 0;
}

/* ---- S5: cascade decode attention ---------------------------------------- */

typedef struct {
    const hkvo_tier *t;
    int64_t j;
} token_ref;

/* [TS 2.A]: decoding reads the dense recent window, the tokens the sparse tier
 * keeps and the condensed slots. Plain softmax attention of one query head over
 * their concatenation. */
int hkvo_attend(const hkvo_dims *d, const void *q, const hkvo_tier *dense,
                const hkvo_tier *sparse, const int32_t *idx, const int32_t *sel_len,
                int32_t bmax, const hkvo_tier *condensed, float *out, float *lse)
{
    if (check_dims(d) || q == NULL || out == NULL || lse == NULL)
        return -1;
    int32_t units = d->B * d->Hkv;
    if (check_tier(dense, units) || check_tier(sparse, units) || check_tier(condensed, units))
        return -1;
    if (sparse && (idx == NULL || sel_len == NULL))
        return -1;
    int32_t G = d->Hq / d->Hkv, D = d->D;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : err)
    for (int32_t u = 0; u < units; ++u) {
        int32_t b = u / d->Hkv, h = u % d->Hkv;
        int32_t W = tier_len(dense, u), C = tier_len(condensed, u);
        int32_t k = sparse ? sel_len[u] : 0;
        int32_t T = W + k + C;
        token_ref *toks = (token_ref *)malloc(sizeof(token_ref) * (size_t)(T > 0 ? T : 1));
        double *s = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double *acc = (double *)malloc(sizeof(double) * (size_t)D);
        if (!toks || !s || !acc) {
            err = -3;
            free(toks);
            free(s);
            free(acc);
            continue;
        }
        int32_t t = 0;
        for (int32_t j = 0; j < W; ++j)
            toks[t++] = (token_ref){dense, j};
        for (int32_t i = 0; i < k; ++i) {
            int32_t j = idx[(int64_t)u * bmax + i];
            if (j < 0 || j >= sparse->len[u])
                err = -1;
            toks[t++] = (token_ref){sparse, j < 0 ? 0 : j};
        }
        for (int32_t j = 0; j < C; ++j)
            toks[t++] = (token_ref){condensed, j};
        for (int32_t g = 0; g < G; ++g) {
            int32_t hq = h * G + g;
            float *o = out + ((int64_t)b * d->Hq + hq) * D;
            if (T == 0) {
                for (int32_t x = 0; x < D; ++x)
                    o[x] = 0.0f;
                lse[(int64_t)b * d->Hq + hq] = -INFINITY;
                continue;
            }
            double M = -INFINITY;
            for (int32_t i = 0; i < T; ++i) {
                s[i] = d->scale * dot_qk(d, q, b, hq, toks[i].t, h, toks[i].j);
                if (s[i] > M)
                    M = s[i];
            }
            double L = 0.0;
            for (int32_t x = 0; x < D; ++x)
                acc[x] = 0.0;
            for (int32_t i = 0; i < T; ++i) {
                double w = exp(s[i] - M);
                int64_t vo = row_off(toks[i].t, b, h, toks[i].j);
                L += w;
                for (int32_t x = 0; x < D; ++x)
                    acc[x] += w * elem(toks[i].t->v, d->dtype, vo + x);
            }
            for (int32_t x = 0; x < D; ++x)
                o[x] = (float)(acc[x] / L);
            lse[(int64_t)b * d->Hq + hq] = (float)(M + log(L));
        }
        free(toks);
        free(s);
        free(acc);
    }
    return err;
}

/* ---- the whole step ------------------------------------------------------- */

int hkvo_step(const hkvo_dims *d, const void *q, const hkvo_tier *dense,
              const hkvo_tier *sparse, const hkvo_tier *condensed, const float *beta,
              float p, const float *p_unit, int32_t bmin, int32_t bmax, float *z,
              int32_t *k, int32_t *idx, float *out, float *lse)
{
    if (check_dims(d) || sparse == NULL)
        return -1;
    int32_t units = d->B * d->Hkv;
    int r = hkvo_score(d, q, sparse, z, sparse->cap);
    if (r == 0)
        r = hkvo_topp(units, z, sparse->cap, sparse->len, beta, p, p_unit, bmin, bmax, k,
                      NULL, NULL, NULL);
    if (r == 0)
        r = hkvo_compact(units, z, sparse->cap, sparse->len, k, bmax, HKVO_PAD_MAX, idx, NULL);
    if (r == 0)
        r = hkvo_attend(d, q, dense, sparse, idx, k, bmax, condensed, out, lse);
    return r;
}

int hkvo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
