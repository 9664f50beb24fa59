/*
 * hkv.h -- C ABI of the B200 (sm_100a) library for the decode-time hot path of
 * HARD-KV's Cascade Cache.
 *
 * Sources named in the comments:
 *   [Abstract] arXiv abstract on the mlsanity.com page "HARD-KV: Head-Adaptive
 *              Regularization for Decoding-time KV Compression".
 *   [TS 2.A]   gist.science Technical Summary of that paper, section 2.A
 *              "Cascade Cache Hierarchy"; [TS 2.B] "Logits Calibration
 *              Mechanism"; [TS 2.C] "System-Aware Index Regularization";
 *              [TS 3] "Key Contributions"; [TS 5] "Significance and Claims".
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * - Memory: the caller owns all memory. Pointers marked "device" must be
 *   device-accessible (cudaMalloc or torch CUDA tensors) on the current device;
 *   pointers marked "host" are host memory. The library never allocates, frees
 *   or synchronises on the compute path (hkv_get_status is the one call that
 *   synchronises). Every compute call is asynchronous on `stream` and can be
 *   captured in a CUDA graph: shapes are static and every length, budget and
 *   temperature that changes from step to step is read on the device
 *   ([TS 2.C] Head-wise Block Manager: static tensor shapes and persistent
 *   pointers; [TS 5] CUDA Graph compatibility over many decoding steps).
 * - A *unit* is one KV head of one sequence, u = b*Hkv + h. Per-unit arrays are
 *   length B*Hkv in that order.
 * - Query head h*G + g (g < G = Hq/Hkv) attends through KV head h.
 * - A tier stores K and V as [B, Hkv, cap, D] with D contiguous and element
 *   strides (stride_b, stride_h, stride_t); rows must start on 16-byte
 *   boundaries (base pointers 16-byte aligned, strides multiples of 8 bf16 or
 *   4 fp32 elements).
 * - Return codes report host-side validation and CUDA launch errors only; a
 *   call that returns an error has launched nothing unless it says otherwise.
 *   Conditions found on the device (a length above its capacity, a bounded
 *   wait that ran out, a negative temperature) set bits in a status word in
 *   the workspace, read by hkv_get_status. No exception crosses the ABI.
 * - Scores and Top-p selection follow one fixed rule: tokens are ordered by
 *   score descending, ties by lower token index (-0 equals +0); the budget is
 *   the fewest tokens whose calibrated mass is at least p, clamped to
 *   [bmin, bmax] and to the tokens present.
 */
#ifndef HKV_H
#define HKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *hkv_stream_t;

typedef enum {
    HKV_OK = 0,
    HKV_ERR_INVALID_ARG = 1,  /* a pointer, shape, stride, alignment or value is invalid */
    HKV_ERR_UNSUPPORTED = 2,  /* valid but not built: D not in {64,128}, G not in {1,2,4,8} */
    HKV_ERR_CUDA = 3,         /* a CUDA runtime call failed (launch, copy, attribute) */
    HKV_ERR_TIMEOUT = 4,      /* hkv_get_status: a bounded device wait ran out */
    HKV_ERR_DEVICE = 5,       /* hkv_get_status: another device-side condition (see flags) */
    HKV_ERR_WORKSPACE = 6     /* workspace pointer missing, misaligned or too small */
} hkv_status;

typedef enum { HKV_BF16 = 0, HKV_F32 = 1 } hkv_dtype;

/* [TS 2.C] Flatten Index: indices regularised to the maximum length or to the
 * sum of the lengths. */
typedef enum {
    HKV_LAYOUT_PAD_MAX = 0,   /* idx[u*bmax + i], rows padded with -1 */
    HKV_LAYOUT_FLAT_SUM = 1   /* idx[offsets[u] + i], offsets[B*Hkv+1] */
} hkv_layout;

/* Device status-word bits (hkv_get_status). */
#define HKV_DEV_LEN_CLAMPED  0x1u  /* a per-unit length exceeded its capacity; clamped */
#define HKV_DEV_TIMEOUT      0x2u  /* a bounded wait ran out; outputs of that call invalid */
#define HKV_DEV_BAD_TEMP     0x4u  /* a negative or NaN inverse temperature; 1 used */
#define HKV_DEV_BAD_INDEX    0x8u  /* an index or budget outside its range; row 0 / a clamp used */
#define HKV_DEV_BAD_P        0x10u /* a NaN per-unit p; p = 1 used */
#define HKV_DEV_SPARSE_FULL  0x20u /* hkv_append: a token left the dense window while the
                                      sparse tier was full, and was dropped */

/* One cache tier ([TS 2.A]: dense recent window, sparse tier, condensed slots). */
typedef struct {
    const void *k;            /* device, [B, Hkv, cap, D] */
    const void *v;            /* device, same shape and strides as k (may be NULL for
                                 calls that read only keys: hkv_score, hkv_compact without
                                 rewrite) */
    int64_t stride_b, stride_h, stride_t;  /* element strides; D is contiguous */
    int32_t cap;              /* token capacity per unit (0 <= len <= cap) */
    const int32_t *len;       /* device [B*Hkv], valid tokens per unit */
} hkv_tier;

/* The problem statement of one decode step of one layer. */
typedef struct {
    int32_t B, Hq, Hkv, D;    /* sequences, query heads, KV heads, head dim (64 or 128) */
    hkv_dtype dtype;          /* element type of q, K, V */
    float scale;              /* logit scale; 0 selects 1/sqrt(D) */
    float p;                  /* Top-p mass ([Abstract]); used when p_unit is NULL */
    int32_t bmin, bmax;       /* budget clamps, 0 <= bmin <= bmax ([TS 2.A] hard limits) */
    hkv_layout layout;        /* compacted index layout */
    const float *inv_temp;    /* device [B*Hkv] Logits Calibration inverse temperature
                                 beta ([TS 2.B]); NULL = 1 everywhere */
    const float *p_unit;      /* device [B*Hkv] per-unit p; NULL = use p */
} hkv_problem;

/* Per-unit cut of the Top-p selection, produced by hkv_topp_select and read by
 * hkv_compact. The selected set is every token whose score is above z_cut, plus
 * the first n_tie tokens (in index order) whose score equals z_cut. */
typedef struct {
    float z_cut;              /* score of the last selected token (0 if k = 0) */
    int32_t n_above;          /* selected tokens scoring above z_cut */
    int32_t n_tie;            /* selected tokens scoring exactly z_cut */
    int32_t kstar;            /* unclamped Top-p budget, or -1 when the clamp decided
                                 k without computing it */
} hkv_cut;

/* Outputs of hkv_step. Optional pointers may be NULL. */
typedef struct {
    int32_t *sel_len;         /* device [B*Hkv], budget k per unit (required) */
    int32_t *idx;             /* device, layout of problem.layout (required):
                                 PAD_MAX [B*Hkv*bmax]; FLAT_SUM [B*Hkv*bmax] capacity */
    int32_t *offsets;         /* device [B*Hkv+1], FLAT_SUM only (required there) */
    float *out;               /* device [B, Hq, D] fp32 attention output (required) */
    float *lse;               /* device [B, Hq] fp32 natural-log sum of exp (optional) */
    float *z;                 /* device [B*Hkv, sparse.cap] fp32 scores (optional) */
    hkv_cut *cut;             /* device [B*Hkv] (optional) */
    float *m;                 /* device [B*Hkv] max score (optional) */
    float *logZ;              /* device [B*Hkv] log of the calibration normaliser (optional) */
    void *k_out, *v_out;      /* device Rewrite Cache rows in the idx layout:
                                 PAD_MAX [B*Hkv, bmax, D]; FLAT_SUM [B*Hkv*bmax, D] (optional,
                                 both or neither) */
    float *beta_fit;          /* device [B*Hkv] (optional): when given, the step fits each
                                 unit's inverse temperature as hkv_attention_entropy +
                                 hkv_fit_temperature define it, writes it here and selects
                                 with it in place of prob->inv_temp */
    float *h_attn;            /* device [B*Hkv] (optional, only with beta_fit): the target
                                 entropies the fit used */
} hkv_step_out;

/* Size in bytes of the workspace the calls below need for this problem and
 * these tier capacities (it depends on shapes only, never on lengths). Host
 * pointers; tiers may be NULL for an empty tier. */
hkv_status hkv_workspace_size(const hkv_problem *prob, const hkv_tier *dense,
                              const hkv_tier *sparse, const hkv_tier *condensed,
                              size_t *bytes);

/* Zero a workspace (asynchronous memset on `stream`). Required once before its
 * first use, and again after a call whose status reported HKV_DEV_TIMEOUT. */
hkv_status hkv_workspace_init(void *ws, size_t bytes, hkv_stream_t stream);

/* S1 Score ([TS 2.B] max-pooled attention logits; [TS 2.A] Tier 2):
 * z[u*z_stride + j] = scale * max_g q[b, h*G+g, :] . K_sparse[b, h, j, :] for
 * j < len[u], fp32 accumulation from bf16/fp32 inputs. q: device [B, Hq, D].
 * z: device, 4-byte aligned; z_stride >= sparse->cap. Entries past len[u] are
 * not written. */
hkv_status hkv_score(const hkv_problem *prob, const void *q, const hkv_tier *sparse,
                     float *z, int64_t z_stride, void *ws, size_t ws_bytes,
                     hkv_stream_t stream);

/* S2 Logits Calibration ([TS 2.B], [TS 3]): per unit m = max_j z_j,
 * Z = sum_j exp(beta (z_j - m)), logZ = ln Z, and optionally
 * P[u*z_stride + j] = exp(beta (z_j - m)) / Z. sparse supplies the lengths
 * (its K/V are not read). m, logZ: device [B*Hkv]; P may be NULL. An empty unit
 * gives m = -inf, logZ = -inf. Z is the exact integer sum of the weights
 * floored to 40-bit fixed point (so it is low by at most n 2^-40, with Z >= 1),
 * exactly as hkv_topp_select and hkv_step sum it. */
hkv_status hkv_calibrate(const hkv_problem *prob, const float *z, int64_t z_stride,
                         const hkv_tier *sparse, float *P, float *m, float *logZ,
                         void *ws, size_t ws_bytes, hkv_stream_t stream);

/* S3 Top-p budget ([Abstract], [TS 2.A], [TS 2.B]): per unit the budget
 * sel_len[u] = min(n, max(bmin, min(k*, bmax))), k* the fewest tokens (score
 * descending, lower index first) whose calibrated mass is at least p, and the
 * cut that identifies the set. Prefix masses and Z are exact sums of the same
 * 40-bit fixed-point weights, so the result does not depend on the order of
 * summation and is deterministic. sparse supplies the lengths.
 * sel_len, cut: device [B*Hkv]. */
hkv_status hkv_topp_select(const hkv_problem *prob, const float *z, int64_t z_stride,
                           const hkv_tier *sparse, int32_t *sel_len, hkv_cut *cut,
                           void *ws, size_t ws_bytes, hkv_stream_t stream);

/* S4 Index Regularization ([TS 2.C] Flatten Index, Rewrite Cache): writes the
 * selected tokens of each unit in ascending index order into idx (layout of
 * prob->layout; PAD_MAX rows padded with -1; FLAT_SUM offsets = exclusive scan
 * of sel_len over units). If k_out and v_out are given, also copies the selected
 * K/V rows bit for bit into them, in the same layout (rows of D elements).
 * sparse supplies len (and K/V for the rewrite). */
hkv_status hkv_compact(const hkv_problem *prob, const float *z, int64_t z_stride,
                       const hkv_tier *sparse, const int32_t *sel_len, const hkv_cut *cut,
                       int32_t *idx, int32_t *offsets, void *k_out, void *v_out,
                       void *ws, size_t ws_bytes, hkv_stream_t stream);

/* S5 Cascade decode attention ([TS 2.A] three tiers; [Abstract]): for each
 * query head, softmax attention (scale * q.k) over dense[0, len) ++
 * sparse[idx_0 .. idx_{k-1}] ++ condensed[0, len), split across all warps of a
 * persistent grid (dense and condensed tokens on one work line, the selected
 * tokens on another) and merged by online softmax in a second kernel. out: device [B, Hq, D] fp32; lse: device [B, Hq] fp32 or
 * NULL. idx/offsets in prob->layout with k = sel_len[u]. An empty token list
 * gives out = 0, lse = -inf. Any tier may be NULL (empty). ws: workspace of
 * hkv_workspace_size bytes, zeroed once by hkv_workspace_init. */
hkv_status hkv_cascade_decode(const hkv_problem *prob, const void *q,
                              const hkv_tier *dense, const hkv_tier *sparse,
                              const int32_t *idx, const int32_t *offsets,
                              const int32_t *sel_len, const hkv_tier *condensed,
                              float *out, float *lse, void *ws, size_t ws_bytes,
                              hkv_stream_t stream);

/* S1..S5 in one call ([TS 2.A] pipeline steps 2 and 3 plus decoding): four
 * kernels on `stream`, each launched as a programmatic dependent of the
 * kernel before it (the first waits for that kernel before reading anything). (1) A persistent streaming kernel scores every sparse
 * token (the same kernel as hkv_score), also writing each token's per-head
 * logits and each unit's score range into the workspace; (2) one CTA per unit
 * (a cluster of four, or two, for units of more than 24576 sparse tokens)
 * calibrates, takes the Top-p budget and the cut, and compacts the unit's
 * indices into PAD_MAX rows; (3) a
 * persistent streaming kernel attends over the dense and condensed tokens
 * (before it waits for (2)) and over the selected tokens, whose rows it reads
 * through the indices ([TS 2.C] Sparse Loading; four V rows per TMA gather
 * when the sparse tier's rows are contiguous and its units back to back)
 * together with the scorer's logits (so their K rows are not read again); (2) and (3) read the tiers'
 * lengths before their waits, so the lengths must be final when the call is
 * made (this library's append and condensation let no dependent start before
 * they end); (4) a merge kernel combines
 * each unit's partial softmax records. A FLAT_SUM layout or
 * k_out/v_out (the Rewrite Cache copy) adds a kernel at the end; out->beta_fit
 * adds one between (1) and (2) that fits each unit's inverse temperature from
 * the scorer's per-head logits and scores (hkv_attention_entropy and
 * hkv_fit_temperature give the same bits), after which (2) selects with it. Scores, budgets,
 * cuts, index rows, m and logZ equal those of the separate calls bit for bit;
 * out and lse agree to a few ulp (hkv_cascade_decode recomputes the logits
 * from K). ws as for hkv_cascade_decode. */
hkv_status hkv_step(const hkv_problem *prob, const void *q, const hkv_tier *dense,
                    const hkv_tier *sparse, const hkv_tier *condensed,
                    const hkv_step_out *out, void *ws, size_t ws_bytes,
                    hkv_stream_t stream);

/* State and thresholds of the trade-off between Rewrite Cache and Sparse
 * Loading ([TS 2.C] Trade-off Management: a Memory-Time Integral weighs the
 * upfront cost of rewriting against the per-step decoding gains, and budget
 * thresholds L_lower and L_upper trigger sparse loading or full rewriting;
 * [TS 4]: the rewrite overhead is amortized within a few decoding steps).
 * Every per-unit array is caller-owned device memory, zero before the first
 * step (all units start in Sparse Loading with no rewrite). */
typedef struct {
    int32_t L_lower, L_upper;  /* budget thresholds (tokens), 0 <= L_lower <= L_upper: a fresh budget
                                  k > L_upper switches the unit to Rewrite Cache, k < L_lower to Sparse
                                  Loading, and a budget in between keeps the unit's mode */
    int64_t mti_cap;           /* memory-time allowance of one rewrite, in row-steps: a rewrite of k
                                  rows serves H(k) = max(1, floor(mti_cap / k)) steps, the step that
                                  made it included */
    int32_t *mode;             /* device [B*Hkv]: 0 Sparse Loading, 1 Rewrite Cache (read, written) */
    int32_t *left;             /* device [B*Hkv]: further steps the unit's rewrite serves (read, written) */
    hkv_tier rewrite;          /* the rewrite buffer: K, V [B, Hkv, cap >= bmax, D] (written), len =
                                  device [B*Hkv] rows it holds (written) */
    int32_t *rw_idx;           /* device [B*Hkv*bmax]: token indices of the rewritten rows (written) */
} hkv_mti;

/* The decode step under the Rewrite Cache / Sparse Loading trigger ([TS 2.C]
 * Rewrite Cache: selected rows moved to contiguous ranges; Sparse Loading: rows
 * read through the indices; Trade-off Management). Per unit u at each call:
 * - left[u] > 0 (the unit reuses its rewrite): the unit is not scored or
 *   selected; its attention runs over dense ++ rewrite rows [0, rewrite.len[u])
 *   ++ condensed, read as contiguous rows; its outputs report sel_len[u] =
 *   rewrite.len[u] and, in idx, the rows' token indices as of the rewrite;
 *   cut, m and logZ are NaN (kstar -1); afterwards left[u] -= 1.
 * - left[u] == 0: the unit is scored, selected and attended exactly as by
 *   hkv_step (Sparse Loading of the fresh selection). Then its mode follows the
 *   trigger on the fresh budget k (above), and under Rewrite Cache its k
 *   selected K and V rows are copied to rewrite rows 0 .. k-1 (bit copies,
 *   token order), rw_idx gets their indices, rewrite.len[u] = k and
 *   left[u] = H(k) - 1; under Sparse Loading rewrite.len[u] = left[u] = 0.
 * Other arguments and outputs as for hkv_step, except that out->k_out/v_out
 * and out->beta_fit must be NULL. At most 1024 units (HKV_ERR_UNSUPPORTED
 * beyond). A rewrite keeps the rows it copied: a token that ages into the
 * sparse tier, or a condensation (hkv_condense) of the unit, takes effect for
 * the unit at its next fresh step; set left[u] = 0 to force one. One more
 * kernel than hkv_step (the trigger and the copies), a cluster of four CTAs
 * per unit. */
hkv_status hkv_step_mti(const hkv_problem *prob, const void *q, const hkv_tier *dense, const hkv_tier *sparse,
                        const hkv_tier *condensed, const hkv_mti *mti, const hkv_step_out *out, void *ws,
                        size_t ws_bytes, hkv_stream_t stream);

/* KV append with the dense-window roll ([TS 2.A] Cascade Cache Hierarchy,
 * pipeline step 1: the new token joins the dense window of recent tokens, and
 * the token that leaves the window moves to the sparse tier). One kernel, one
 * warp per unit. Per unit u = b*Hkv + h, with W = dense->len[u],
 * n = sparse->len[u], and the window a ring of Wc = dense->cap slots whose
 * oldest token sits at slot dense_head[u]:
 *   - W < Wc: the new row goes to dense slot W; dense->len[u] = W + 1.
 *   - W == Wc > 0: the row at slot dense_head[u] leaves the window and the new
 *     row takes its slot; dense_head[u] = (dense_head[u] + 1) mod Wc.
 *   - Wc == 0 (dense NULL or empty): the new row itself leaves at once.
 *   - a row that leaves goes to sparse slot n and sparse->len[u] = n + 1; if
 *     n == sparse->cap it is dropped, dropped[u] = 1 and the status word gets
 *     HKV_DEV_SPARSE_FULL.
 * Rows are copied bit for bit, K and V alike. The sparse tier thus holds the
 * aged-out tokens in age order, which is the token order every other call of
 * this library scores, selects and compacts in. Start a window with len 0 and
 * head 0; a window filled some other way must set head to its oldest slot.
 * - k_new, v_new: device [B, Hkv, D] contiguous, 16-byte aligned, element type
 *   of prob->dtype; must not overlap the tiers.
 * - dense, sparse: tiers as elsewhere (either may be NULL or empty); THIS CALL
 *   WRITES through their k, v and len pointers (declared const in hkv_tier for
 *   the calls that only read them). Both need v.
 * - dense_head: device int32 [B*Hkv], read and written; required when the
 *   dense tier has slots, else may be NULL.
 * - dropped: device int32 [B*Hkv] or NULL; receives 0 or 1 per unit.
 * - Only prob's B, Hkv, D and dtype are used (the rest must still validate).
 * - A unit whose lengths are outside [0, cap] or whose head is outside
 *   [0, Wc) is left untouched and sets HKV_DEV_LEN_CLAMPED or
 *   HKV_DEV_BAD_INDEX.
 * - ws: any workspace of at least 256 bytes (256-byte aligned, zeroed once);
 *   only its status word is used, so the step's workspace serves. */
hkv_status hkv_append(const hkv_problem *prob, const void *k_new, const void *v_new,
                      const hkv_tier *dense, int32_t *dense_head, const hkv_tier *sparse,
                      int32_t *dropped, void *ws, size_t ws_bytes, hkv_stream_t stream);

/* Fitted temperature, part 1 ([TS 2.A] Tier 2: budgets from attention
 * entropy; [TS 3]: calibration onto the raw attention distribution): per unit
 * the mean, over the G query heads of its group, of the entropy (natural log)
 * of each head's raw attention softmax_j(scale * q_g . k_j) over the sparse
 * tokens j < len[u]; 0 for an empty unit. Two kernels: the scorer (the same as
 * hkv_score, here writing each token's per-head logits into the workspace)
 * and a cluster of two CTAs per unit summing in double precision.
 * q: device [B, Hq, D]; h: device [B*Hkv] fp32. */
hkv_status hkv_attention_entropy(const hkv_problem *prob, const void *q, const hkv_tier *sparse,
                                 float *h, void *ws, size_t ws_bytes, hkv_stream_t stream);

/* Upper end of the fitted inverse temperature. */
#define HKV_FIT_BETA_MAX 64.0f

/* Fitted temperature, part 2 ([TS 2.B] calibration "by adjusting the
 * temperature"): per unit the inverse temperature beta in [0, HKV_FIT_BETA_MAX]
 * at which the calibrated distribution softmax(beta z) of the unit's metric
 * z[u*z_stride + j], j < len[u], has entropy h_target[u]. That entropy does
 * not increase with beta, so the root is unique when z is not constant; it is
 * found by Newton steps inside a shrinking bracket, sums in double precision.
 * A target at or above ln(len) gives 0, one below the entropy at
 * HKV_FIT_BETA_MAX gives HKV_FIT_BETA_MAX, a unit with len <= 1 or constant
 * scores gives 1, and a NaN target gives 1 and HKV_DEV_BAD_TEMP. z may be any
 * metric (max-pooled logits from hkv_score, similarity scores, ...); the
 * result can be passed as prob->inv_temp. One CTA per unit.
 * z: device fp32, z_stride >= sparse->cap; h_target, beta: device [B*Hkv]. */
hkv_status hkv_fit_temperature(const hkv_problem *prob, const float *z, int64_t z_stride,
                               const hkv_tier *sparse, const float *h_target, float *beta,
                               void *ws, size_t ws_bytes, hkv_stream_t stream);

/* Condensed-tier formation ([TS 2.A] Tier 3: "the oldest blocks are further
 * compressed into constant-sized storage via eviction or weighted merging";
 * pipeline step 4, "eviction or merging of the oldest blocks"). One kernel, a
 * cluster of four CTAs per unit. A unit u whose sparse tier holds
 * n >= max(trigger, block) tokens gives up its oldest `block` tokens (sparse
 * slots 0 .. block-1: the tier is in age order, as hkv_append keeps it); they
 * become ONE condensed slot, written after the existing slots:
 *   HKV_CONDENSE_MERGE: the slot's K and V rows are the weighted means of the
 *     block's rows, weighted by the tokens' calibrated probabilities
 *     a_j = exp(beta_u (z_j - m_u) - logZ_u) under the step's scores (beta_u
 *     from prob->inv_temp, 1 when NULL), and the slot's weight is sum_j a_j. A
 *     full condensed tier first merges its two oldest slots the same way
 *     (weighted by their weights; the result weighs their sum) and moves the
 *     later slots down; a tier of one slot folds the block into that slot.
 *   HKV_CONDENSE_EVICT: the slot is a bit copy of the block's most important
 *     token (largest z_j, the older one on ties), weighing a_j; the rest of
 *     the block is dropped. A full condensed tier first drops its oldest slot.
 * Weights that sum to zero, or no scores (z, m, logZ all NULL), mean equal
 * weights (and EVICT keeps the oldest token). Means are float64 sums in slot
 * order, each product and sum rounded separately, divided once and rounded
 * once to the element type (nearest, ties to even; bf16 straight from the
 * double). The sparse tier then moves down by `block` rows (age order kept)
 * and its length drops by `block`; a condensed tier of capacity 0 just loses
 * the block. The cost is a read and a write of the unit's remaining sparse
 * rows; it is paid once per `block` appends when the call runs after each
 * step with trigger = the sparse capacity.
 * - sparse, condensed: tiers as elsewhere (condensed may be NULL or empty);
 *   THIS CALL WRITES through their k, v and len pointers.
 * - cond_w: device fp32 [B*Hkv, condensed->cap], the slots' weights, read and
 *   written (required when the condensed tier has slots; start with zeros or
 *   the weights of slots filled some other way).
 * - z (z_stride >= sparse->cap), m, logZ: device fp32, the scores of the
 *   sparse tier and each unit's max and log normaliser from the last step
 *   (hkv_step's z, m and logZ outputs); all three or none.
 * - block: 1 .. min(HKV_CONDENSE_MAX_BLOCK, sparse->cap); trigger >= 0.
 * - done: device int32 [B*Hkv] or NULL; 1 where the unit gave up a block.
 * - A unit whose lengths are outside [0, cap] is left as it is and sets
 *   HKV_DEV_LEN_CLAMPED; a negative or NaN inverse temperature uses 1 and
 *   sets HKV_DEV_BAD_TEMP.
 * - ws: any workspace of at least 256 bytes (only its status word is used). */
typedef enum { HKV_CONDENSE_MERGE = 0, HKV_CONDENSE_EVICT = 1 } hkv_condense_policy;
#define HKV_CONDENSE_MAX_BLOCK 8192
hkv_status hkv_condense(const hkv_problem *prob, const hkv_tier *sparse, const hkv_tier *condensed,
                        float *cond_w, const float *z, int64_t z_stride, const float *m, const float *logZ,
                        int32_t block, int32_t trigger, hkv_condense_policy policy, int32_t *done,
                        void *ws, size_t ws_bytes, hkv_stream_t stream);

/* Capacity, in bytes, of the device scratch array behind
 * hkv_cascade_decode_noalloc (one array per GPU that loads the library, held
 * until the process exits). */
#define HKV_NOALLOC_SCRATCH_BYTES (4u << 20)

/* S5 without a caller-supplied workspace. No counterpart in the paper: this is
 * an integration aid. Some callers cannot allocate device memory at the point
 * where they decode: a serving engine that hands nearly all HBM to its KV-cache
 * pool at start-up and forbids allocation on the decode path, or a plugin
 * whose enqueue hook may not allocate and has no workspace to offer. This call
 * computes exactly what hkv_cascade_decode computes, with the same kernel and
 * the same arguments minus ws/ws_bytes, and allocates nothing (no cudaMalloc,
 * no cudaFree, no allocating library routine): its scratch is a fixed device
 * array of HKV_NOALLOC_SCRATCH_BYTES bytes inside the library.
 * - Size limit: the scratch holds a status word, a few words per unit and
 *   two attention records of 4*G*(D+2) bytes per streaming warp and per unit
 *   (5.2 MB for a full 148-SM grid at bf16, D = 128, G = 4, 64 units). When the
 *   array cannot hold the records of a full grid, fewer CTAs run (117 CTAs in
 *   that example); a problem with too many units for even one CTA (about 1000
 *   units at G = 4, D = 128) is refused with HKV_ERR_WORKSPACE before anything
 *   is launched: use hkv_cascade_decode with a workspace for those.
 * - Set-up: a call made outside stream capture looks up the array's device
 *   address in the current context (the first one on a device also loads the
 *   module and sets the kernel's shared-memory attribute); a call under
 *   capture reuses the address found by the last call outside capture on that
 *   device. So make the first call on each device, and the first after a
 *   cudaDeviceReset (which also discards the array's contents), outside any
 *   stream capture.
 * - Sharing: every call on a device uses the same array, which keeps the last
 *   call's contents. Each call zeroes the one word that must start at zero
 *   (the status word) on `stream` before its kernels run; everything else is
 *   written before it is read. Calls that overlap on the GPU (other
 *   streams, other host threads) race on the array and give undefined results:
 *   serialise them.
 * - status: device pointer to one uint32 or NULL; when given it receives this
 *   call's HKV_DEV_* bits (stream-ordered copy after the kernel).
 * Other arguments, layouts and return codes as for hkv_cascade_decode. */
hkv_status hkv_cascade_decode_noalloc(const hkv_problem *prob, const void *q,
                                      const hkv_tier *dense, const hkv_tier *sparse,
                                      const int32_t *idx, const int32_t *offsets,
                                      const int32_t *sel_len, const hkv_tier *condensed,
                                      float *out, float *lse, uint32_t *status,
                                      hkv_stream_t stream);

/* Every compute call takes a workspace `ws` of at least hkv_workspace_size
 * bytes (256-byte aligned, zeroed once by hkv_workspace_init); its first word
 * is the device status word. Calls that overlap on the GPU need separate
 * workspaces. */

/* Read and clear the device status word of a workspace. Synchronises `stream`.
 * *flags (host, may be NULL) receives the HKV_DEV_* bits. Returns HKV_OK when
 * no bit is set, HKV_ERR_TIMEOUT when HKV_DEV_TIMEOUT is set, else
 * HKV_ERR_DEVICE. */
hkv_status hkv_get_status(void *ws, uint32_t *flags, hkv_stream_t stream);

/* Upper bound, in nanoseconds, of every spin-wait inside the library's kernels
 * (default 1e9). Takes effect at the next launch. */
hkv_status hkv_set_wait_limit_ns(uint64_t ns);

/* Kernel timeline, a measurement aid: while on (it takes effect at the next
 * launch), the step's kernels record, in the workspace they run with, the
 * earliest start and the latest end of each kernel kind (device global
 * timer, nanoseconds; one atomic per CTA at each end). Kinds: 0 scoring,
 * 1 per-unit selection and compaction, 2 attention, 3 merge, 4 layout (FLAT_SUM
 * rows, Rewrite Cache copies), 5 fitted temperature, 6 the rewrite trigger. */
#define HKV_TL_KINDS 7
hkv_status hkv_set_timeline(int32_t on);

/* Read and clear the timeline of a workspace. Synchronises `stream`.
 * start_end: host [2*HKV_TL_KINDS], start then end per kind; 0 and 0 for a
 * kind that did not run since the last read (or since hkv_workspace_init). */
hkv_status hkv_read_timeline(void *ws, uint64_t *start_end, hkv_stream_t stream);

/* Fault injection for tests: when nonzero, the streaming kernels (scoring and
 * attention, hkv_step included) never arm their copy stages, so each consumer's
 * bounded wait runs out, the kernel returns, and the status word gets
 * HKV_DEV_TIMEOUT; results of such a call are undefined. Takes effect at the
 * next launch. */
hkv_status hkv_debug_withhold_publish(int32_t on);

/* Kernel launches this library has issued in this process (all devices). */
uint64_t hkv_launch_count(void);

/* Human-readable name of a status code (static string). */
const char *hkv_status_string(hkv_status s);

#ifdef __cplusplus
}
#endif
#endif /* HKV_H */
