/*
 * hkv_oracle.h -- CPU oracle for one HARD-KV Cascade Cache decode step.
 *
 * TEST INFRASTRUCTURE ONLY. The test suite, the package smoke check and the
 * benchmark's CPU-baseline leg are the only users. The CUDA library shares no
 * code, header or constant with this oracle, and neither includes the other.
 *
 * All pointers are HOST pointers. Element strides are in elements. bf16 data
 * is passed as its raw 16-bit patterns (uint16). A unit u = b*Hkv + h is one
 * KV head of one sequence. Functions return 0 on success and a negative code
 * on a bad argument or a NaN score (the oracle refuses NaN scores).
 */
#ifndef HKV_ORACLE_H
#define HKV_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { HKVO_BF16 = 0, HKVO_F32 = 1 };
enum { HKVO_PAD_MAX = 0, HKVO_FLAT_SUM = 1 };

typedef struct {
    const void *k, *v;       /* [B, Hkv, cap, D] with element strides below   */
    int64_t sb, sh, st;      /* strides of b, h, token; D is contiguous         */
    int32_t cap;             /* token capacity per unit                         */
    const int32_t *len;      /* [B*Hkv] valid tokens per unit                   */
} hkvo_tier;

typedef struct {
    int32_t B, Hq, Hkv, D;
    int32_t dtype;           /* HKVO_BF16 or HKVO_F32, for q, K and V           */
    double scale;            /* logit scale                                     */
} hkvo_dims;

/* S1: z[u*zcap + j] = fl32(scale * max_g q_g . k_j), j < len[u]. */
int hkvo_score(const hkvo_dims *d, const void *q, const hkvo_tier *sp,
               float *z, int32_t zcap);

/* S2: m[u], logZ[u] and (optional) P[u*zcap + j]. beta: [B*Hkv] or NULL (=1). */
int hkvo_calibrate(int32_t units, const float *z, int32_t zcap, const int32_t *len,
                   const float *beta, float *P, float *m, float *logZ);

/* S3: k[u] (clamped budget), kstar[u] (unclamped) and the oracle masses
 * c_before[u] = C_{k*-1}, c_at[u] = C_{k*} (0 when undefined). p_unit: [units]
 * or NULL (use p). Optional outputs may be NULL. */
int hkvo_topp(int32_t units, const float *z, int32_t zcap, const int32_t *len,
              const float *beta, float p, const float *p_unit, int32_t bmin,
              int32_t bmax, int32_t *k, int32_t *kstar, double *c_before,
              double *c_at);

/* S4: the top-k set of each unit (k = sel_len[u]) in ascending token order.
 * PAD_MAX: idx[u*bmax + i], -1 padded. FLAT_SUM: rows back to back and
 * offsets[units+1]. */
int hkvo_compact(int32_t units, const float *z, int32_t zcap, const int32_t *len,
                 const int32_t *sel_len, int32_t bmax, int32_t layout,
                 int32_t *idx, int32_t *offsets);

/* S4 (Rewrite Cache): kc/vc[u, i, :] = K/V[u, idx[u*bmax+i], :] for i < sel_len,
 * bit copies, into [units, bmax, D] contiguous buffers. */
int hkvo_gather(const hkvo_dims *d, const hkvo_tier *sp, const int32_t *idx,
                const int32_t *sel_len, int32_t bmax, void *kc, void *vc);

/* S5: out[B, Hq, D], lse[B, Hq] over dense ++ sparse[idx] ++ condensed. Any tier
 * may be NULL (empty). idx uses the PAD_MAX layout with row length bmax. */
int hkvo_attend(const hkvo_dims *d, const void *q, const hkvo_tier *dense,
                const hkvo_tier *sparse, const int32_t *idx, const int32_t *sel_len,
                int32_t bmax, const hkvo_tier *condensed, float *out, float *lse);

/* S1..S5 in order: writes z (zcap = sparse cap), k, idx (PAD_MAX), out, lse. */
int hkvo_step(const hkvo_dims *d, const void *q, const hkvo_tier *dense,
              const hkvo_tier *sparse, const hkvo_tier *condensed, const float *beta,
              float p, const float *p_unit, int32_t bmin, int32_t bmax, float *z,
              int32_t *k, int32_t *idx, float *out, float *lse);

/* Number of OpenMP threads the oracle uses (1 when built without OpenMP). */
int hkvo_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
