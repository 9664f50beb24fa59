// hkv_api.cu -- kernels and C ABI of the HARD-KV Cascade Cache decode step.
//
// Sources: [Abstract] = arXiv abstract on the mlsanity.com page "HARD-KV:
// Head-Adaptive Regularization for Decoding-time KV Compression"; [TS 2.A],
// [TS 2.B], [TS 2.C] = sections of the gist.science Technical Summary of that
// paper ("Cascade Cache Hierarchy", "Logits Calibration Mechanism",
// "System-Aware Index Regularization").
//
// One decode step (hkv_step) is four kernels on the caller's stream, the last
// three launched as programmatic dependents so that their launch and prologue
// overlap the previous kernel's tail:
//   1. k_score_stream -- S1: every sparse-tier key scored once (streaming);
//   2. k_unit         -- S2-S4: per unit, calibration + Top-p budget + cut,
//                        then the order-preserving compaction of the indices;
//   3. k_attn_stream  -- S5: attention over dense ++ selected ++ condensed,
//                        one online-softmax record per warp and unit part;
//   4. k_merge        -- S5: each unit's records combined per query head.
// FLAT_SUM layouts and the Rewrite Cache copy add k_flatten. hkv_append
// (k_append, at the end of this file) adds each step's new token to the dense
// window and moves the displaced one into the sparse tier.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "hkv_kernels.cuh"

namespace hkv {

// Trace slots (builds with -DHKV_TRACE only): per unit u of the per-unit
// kernel, TR_SEL + 16u + i: 0 start, 1 sweep 1 done, 2 sweep 2 done, 3 cut
// found, 4 range known, 5 compacted, 6 scores staged, 7 rank bin found,
// 8 mass through it summed, 9 count bin found, 10 bin sorted, 11 results
// written; per streaming warp g,
// TR_SW + 4g (scoring) or TR_AW + 4g (attention) + i: 0 pipeline start,
// 1 first stage landed, 2 pipeline done, 3 kernel entry (attention).
// Per unit u of the fitting kernel, TR_FIT + 16u + i: 0 start, 1 entropy
// done, 2 scores staged, 3 beta found; 4 holds the number of evaluations.
// Per unit u of the merge kernel, TR_MRG + 2u: 0 start, 1 done.
// Per attention warp g, TR_AB + 2g: line B start (after the wait and its
// layout), line B done; TR_LB + 4g: line B's pipeline
// (first landing, end, and the stages at TRACE_STAGES + 8 (TR_LB + 4g)).
[[maybe_unused]] constexpr int TR_SEL = 250000, TR_SW = 0, TR_AW = 20000, TR_FIT = 240000, TR_MRG = 260000,
                               TR_AB = 30000, TR_LB = 8000;

// =============================================================================
// Kernels
// =============================================================================

// S1 ([TS 2.B] max-pooled logits over the query group; [TS 2.A] Tier 2):
// persistent streaming scorer over the capacity rows of all units.
template <int ES, int D, int G>
__global__ void __launch_bounds__(sc_nw(G) * 32, 1) k_score_stream(const __grid_constant__ Params P)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    using Job = ScoreJob<ES, D, G>;
    auto &sm = *reinterpret_cast<typename Job::Smem *>(smem_raw);
    const Ctl c = make_ctl(P);
    ring_init(sm.ring);
    allow_dependents();
    wait_prior_grid();  // the previous kernel's results are visible from here on
    const int64_t NW = (int64_t)gridDim.x * Job::NW;
    const int64_t g = (int64_t)blockIdx.x * Job::NW + (threadIdx.x >> 5);
    tl_start(P.tl, TL_SCORE);
    const bool prefix = P.units <= PREFIX_CAP;
    const int64_t T = prefix ? score_prologue<Job::NW * 32>(P, c, sm.line, sm.red)
                             : (int64_t)P.units * P.sparse.cap;
    Job job(P, c, sm.ring, prefix ? &sm.line : nullptr, T, g, NW);
    HKV_TRACE_WARP(TR_SW + 4 * (int)g);
    if (!job.run_static_share())
        warp_pipeline(job, sm.ring, c, TR_SW + 4 * (int)g);
    tl_end(P.tl, TL_SCORE);
}

// S5 ([TS 2.A] cascade decode over the three tiers; [TS 2.C] Sparse Loading):
// persistent streaming attention over line A (dense and condensed tokens, and
// the rows of reused rewrites), before the wait for the selection, then line B
// (the selected sparse tokens); writes one record per warp and unit and line.
template <int ES, int D, int G>
__global__ void __launch_bounds__(AT_NW * 32, 1) k_attn_stream(const __grid_constant__ Params P)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ unsigned long long red[AT_NW];
    using SM = AttnSmem<ES, D, G>;
    SM &sm = *reinterpret_cast<SM *>(smem_raw);
    const Ctl c = make_ctl(P);
    ring_init(sm.ring);
    allow_dependents();
    tl_start(P.tl, TL_ATTN);
    // line A (dense, reused rewrite and condensed tokens) needs only the
    // inputs, so it runs before the wait, alongside the selection kernel
    AttnLens lens;
    attn_read_lengths(P, c, lens);
    const AttnLine A = attn_prologue_a<ES, D, G>(P, sm, red, lens);
    const int64_t g = (int64_t)blockIdx.x * AT_NW + (threadIdx.x >> 5);
    AttnJob<ES, D, G> job(P, c, sm, A, g);
    HKV_TRACE_WARP(TR_AW + 4 * (int)g);
    const uint32_t used = warp_pipeline(job, sm.ring, c, TR_AW + 4 * (int)g);
    // line B (the selected tokens) after the selection
    __syncthreads();
    wait_prior_grid();
    HKV_TRACE_WARP(TR_AW + 4 * (int)g + 3);
    job.begin_line_b(attn_prologue_b<ES, D, G>(P, sm, c, red, lens, A));
    HKV_TRACE_WARP(TR_AB + 2 * (int)g);
    warp_pipeline(job, sm.ring, c, TR_LB + 4 * (int)g, used);
    HKV_TRACE_WARP(TR_AB + 2 * (int)g + 1);
    tl_end(P.tl, TL_ATTN);
}

// S5 merge: out and lse of each (unit, query head) from the unit's records on
// both attention lines, in slot order. Warp w takes head w % G and the
// (w / G)-th of merge_split(G) contiguous parts of the records; the parts of a
// head are then combined in part order.
template <int D, int G>
__global__ void __launch_bounds__(MERGE_WARPS * 32, 1) k_merge(const __grid_constant__ Params P)
{
    constexpr int S = merge_split(G), DPL = D / 32;
    __shared__ float pm[MERGE_WARPS], pl[MERGE_WARPS], po[MERGE_WARPS][D];
    allow_dependents();
    const int u = blockIdx.x;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, g = w % G, part = w / G;
    wait_prior_grid();
    HKV_TRACE_AT(TR_MRG + 2 * u);
    tl_start(P.tl, TL_MERGE);
    const int4 r = __ldcg(reinterpret_cast<const int4 *>(P.rec_range) + u);
    const int na = r.y >= r.x ? r.y - r.x + 1 : 0, nb = r.w >= r.z ? r.w - r.z + 1 : 0;
    const int tot = na + nb;
    float M, L, O[DPL];
    merge_records<D, G>(P, g, r.x, na, r.z, part * tot / S, (part + 1) * tot / S, M, L, O);
#pragma unroll
    for (int e = 0; e < DPL; ++e)
        po[w][lane * DPL + e] = O[e];
    if (lane == 0) {
        pm[w] = M;
        pl[w] = L;
    }
    __syncthreads();
    if (part == 0) {
        for (int q = 1; q < S; ++q) {
            const int x = q * G + g;
            const float mq = pm[x];
            if (mq == -INFINITY)
                continue;
            const float Mn = fmaxf(M, mq);
            const float a = (M == -INFINITY) ? 0.0f : ex2(M - Mn);
            const float f = ex2(mq - Mn);
            L = L * a + pl[x] * f;
#pragma unroll
            for (int e = 0; e < DPL; ++e)
                O[e] = O[e] * a + po[x][lane * DPL + e] * f;
            M = Mn;
        }
        // no tokens at all: out 0, lse -inf
        const int b = u / P.Hkv, h = u % P.Hkv;
        const int hq = h * G + g;
        float *orow = P.out + ((int64_t)b * P.Hq + hq) * D + lane * DPL;
#pragma unroll
        for (int e = 0; e < DPL; ++e)
            orow[e] = (M == -INFINITY) ? 0.0f : O[e] / L;
        if (lane == 0 && P.lse != nullptr)
            P.lse[(int64_t)b * P.Hq + hq] = (M == -INFINITY) ? -INFINITY : (M + log2f(L)) * 0.6931471805599453f;
    }
    HKV_TRACE_AT(TR_MRG + 2 * u + 1);
    tl_end(P.tl, TL_MERGE);
}

// Rewrite Cache ([TS 2.C]): copy the k selected K/V rows of unit u, listed in
// `row`, to rows dst_row0 .. dst_row0 + k - 1 of k_out / v_out.
__device__ void rewrite_rows(const Params &P, int u, const int32_t *row, int k, int64_t dst_row0, int es,
                             const Ctl &c, int n_sparse)
{
    const int b = u / P.Hkv, h = u % P.Hkv;
    const int vec_per_row = P.D * es / 16;
    const int64_t total = (int64_t)k * vec_per_row;
    for (int64_t i = threadIdx.x; i < total; i += NT) {
        const int r = (int)(i / vec_per_row), x = (int)(i % vec_per_row);
        int j = __ldcg(row + r);
        if (j < 0 || j >= n_sparse) {
            raise_flag(c, HKV_DEV_BAD_INDEX);
            j = 0;
        }
        const int64_t src = ((int64_t)b * P.sparse.sb + (int64_t)h * P.sparse.sh + (int64_t)j * P.sparse.st) * es;
        const int64_t dst = (dst_row0 + r) * (int64_t)P.D * es;
        reinterpret_cast<uint4 *>(P.k_out + dst)[x] = __ldcs(reinterpret_cast<const uint4 *>(P.sparse.k + src) + x);
        reinterpret_cast<uint4 *>(P.v_out + dst)[x] = __ldcs(reinterpret_cast<const uint4 *>(P.sparse.v + src) + x);
    }
}

// Start of unit u in the FLAT_SUM layout: the budgets of the units before it.
__device__ int64_t flat_offset(const Params &P, int u, unsigned long long *red)
{
    unsigned long long part = 0;
    for (int i = threadIdx.x; i < u; i += NT)
        part += (unsigned long long)max(0, __ldcg(P.sel_len + i));
    return (int64_t)block_sum_u64<NT>(part, red);
}

__device__ __forceinline__ void write_offsets(const Params &P, int u, int64_t off)
{
    if (threadIdx.x == 0) {
        P.offsets[u] = (int32_t)off;
        if (u == P.units - 1)
            P.offsets[P.units] = (int32_t)(off + max(0, __ldcg(P.sel_len + u)));
    }
}

// S2-S4 of unit u, scores at zu (in shared memory when ZS).
// zg_stage (ZS only): the unit's scores are still in global memory there and
// the fast path stages them during its first sweep. zs_in_flight (ZS only):
// they are landing in shared memory from this thread's cp.async copies.
template <int ES, bool ZS>
__device__ __forceinline__ void unit_work(const Params &P, USmem &sm, const Ctl &c, int u, int n, const float *zu,
                                          const float *zg_stage = nullptr, bool zs_in_flight = false)
{
    int k, n_tie;
    uint32_t key;
    if (P.do_select) {
        float m, zlo;
        if (P.have_range) {
            // the scorer's range words of the unit (key 0: no score), reset
            // for the next step once read (zs_in_flight: k_unit has put them
            // in sm.redf already)
            if (threadIdx.x == 0) {
                if (!zs_in_flight) {
                    const uint32_t kmax = __ldcg(P.urange + 2 * u), kmin = __ldcg(P.urange + 2 * u + 1);
                    sm.redf[0] = kmax ? ord_val(kmax) : -INFINITY;
                    sm.redf[1] = kmin ? ord_val(~kmin) : INFINITY;
                }
                P.urange[2 * u] = 0;
                P.urange[2 * u + 1] = 0;
            }
            __syncthreads();
            m = sm.redf[0];
            zlo = sm.redf[1];
            __syncthreads();
        } else {
            unit_range<ZS>(zu, n, &m, &zlo, sm);
        }
        HKV_TRACE_AT(TR_SEL + 16 * u + 4);
        const float beta = unit_beta(P, u, c), pu = unit_p(P, u, c);
        const auto publish = [&](const Selection &s) {
            if (threadIdx.x == 0) {
                P.sel_len[u] = s.k;
                if (P.cut)
                    P.cut[u] = s.cut;
                if (P.m_out)
                    P.m_out[u] = m;
                if (P.logZ_out)
                    P.logZ_out[u] = n > 0 ? (float)log(s.Z()) : -INFINITY;
            }
        };
        if constexpr (ZS) {
            // selection and PAD_MAX compaction in one go (hkv_step)
            Selection s;
            if (P.do_compact &&
                select_compact_fast(zu, n, m, zlo, beta, pu, P.bmin, P.bmax, sm, s, P.idx + (int64_t)u * P.bmax,
                                    P.bmax, TR_SEL + 16 * u, zg_stage, zs_in_flight)) {
                publish(s);
                HKV_TRACE_AT(TR_SEL + 16 * u + 5);
                return;
            }
        }
        const Selection s = select_unit<ZS>(zu, n, m, zlo, beta, pu, P.bmin, P.bmax, sm, TR_SEL + 16 * u);
        k = s.k;
        key = s.key;
        n_tie = s.cut.n_tie;
        publish(s);
        HKV_TRACE_AT(TR_SEL + 16 * u + 11);
    } else {
        k = __ldcg(P.sel_len + u);
        const hkv_cut ct = P.cut[u];
        if (k < 0 || k > n || k > P.bmax || ct.n_above < 0 || ct.n_tie < 0 || ct.n_above + ct.n_tie != k) {
            raise_flag(c, HKV_DEV_BAD_INDEX);
            k = 0;
        }
        key = k > 0 ? score_key(ct.z_cut) : 0u;
        n_tie = ct.n_tie;
    }
    if (!P.do_compact)
        return;
    const bool flat = P.layout == HKV_LAYOUT_FLAT_SUM && !P.do_select;
    int64_t off = (int64_t)u * P.bmax;
    if (flat) {
        off = flat_offset(P, u, sm.red);
        write_offsets(P, u, off);
    }
    int32_t *row = P.idx + off;
    compact_unit<ZS>(zu, n, key, n_tie, k, row, flat ? k : P.bmax, sm.red, TR_SEL + 16 * u);
    HKV_TRACE_AT(TR_SEL + 16 * u + 5);
    if (P.k_out != nullptr && !P.do_select) {
        __syncthreads();
        rewrite_rows(P, u, row, k, off, ES, c, n);
    }
}

// A unit that reuses its rewrite this step (hkv_step_mti): its step outputs
// describe the rewrite's rows (their token indices as of the rewrite), which
// the attention reads from the rewrite buffer. Its cut, m and logZ are not
// computed (NaN; kstar -1).
__device__ void mti_reuse_outputs(const Params &P, const Ctl &c, int u)
{
    int k = tier_len(P.rw, u, c);
    if (k > P.bmax) {
        raise_flag(c, HKV_DEV_BAD_INDEX);
        k = P.bmax;
    }
    int32_t *row = P.idx + (int64_t)u * P.bmax;
    for (int i = threadIdx.x; i < P.bmax; i += NT)
        row[i] = i < k ? __ldcg(P.rw_idx + (int64_t)u * P.bmax + i) : -1;
    if (threadIdx.x == 0) {
        P.sel_len[u] = k;
        if (P.cut)
            P.cut[u] = hkv_cut{__int_as_float(0x7fc00000), 0, 0, -1};
        if (P.m_out)
            P.m_out[u] = __int_as_float(0x7fc00000);
        if (P.logZ_out)
            P.logZ_out[u] = __int_as_float(0x7fc00000);
    }
}

// S2-S4 per unit, one CTA per (sequence, KV head). Units of up to ZSTAGE
// tokens work on a copy of their scores in shared memory.
//  do_select  ([TS 2.B] calibration, [Abstract]/[TS 2.A] Top-p budget with the
//             hard limits): writes sel_len, cut, m, logZ. With have_range the
//             unit's score range comes from the scorer's range words.
//  do_compact ([TS 2.C] Flatten Index): writes the unit's indices in score
//             order from the cut -- PAD_MAX rows, or FLAT_SUM (standalone) --
//             and, standalone, the Rewrite Cache copy when k_out is given.
template <int ES>
__global__ void __launch_bounds__(NT, 1) k_unit(const __grid_constant__ Params P)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    USmem &sm = *reinterpret_cast<USmem *>(smem_raw);
    const Ctl c = make_ctl(P);
    const int u = blockIdx.x;
    allow_dependents();
    // the unit's length is an input of the step (no kernel of the step writes
    // it, and the kernels that do, the append and the condensation, let their
    // dependents start only when they end): read before the wait
    const int n = tier_len(P.sparse, u, c);
    wait_prior_grid();
    HKV_TRACE_AT(TR_SEL + 16 * u);
    tl_start(P.tl, TL_UNIT);
    const float *zg = P.z + (int64_t)u * P.z_stride;
    // hkv_step: with the range known and every unit short enough to stage,
    // the range words are requested first, then the scores' copy into shared
    // memory (which the loads would otherwise queue behind)
    const bool early = P.have_range && P.do_select && P.do_compact && P.sparse.cap <= ZSTAGE &&
                       (reinterpret_cast<uintptr_t>(zg) & 15) == 0;
    uint32_t kmax = 0, kmin = 0;
    if (early && threadIdx.x == 0) {
        kmax = __ldcg(P.urange + 2 * u);
        kmin = __ldcg(P.urange + 2 * u + 1);
    }
    if (early) {
        stage_scores_async(zg, P.sparse.cap, sm.zs);
        if (threadIdx.x == 0) {
            sm.redf[0] = kmax ? ord_val(kmax) : -INFINITY;
            sm.redf[1] = kmin ? ord_val(~kmin) : INFINITY;
        }
    }
    if (P.mti_left != nullptr && __ldcg(P.mti_left + u) > 0) {
        if (early)
            cp_async_wait_all();
        mti_reuse_outputs(P, c, u);  // the unit reuses its rewrite: nothing to select
    } else if (early) {
        unit_work<ES, true>(P, sm, c, u, n, sm.zs, nullptr, true);
    } else if (P.have_range && P.do_select && P.do_compact && n <= ZSTAGE) {
        // hkv_step: the range is known, so the first sweep stages the scores
        unit_work<ES, true>(P, sm, c, u, n, sm.zs, zg);
    } else {
        const bool staged = stage_scores(zg, n, sm);
        HKV_TRACE_AT(TR_SEL + 16 * u + 6);
        if (staged)
            unit_work<ES, true>(P, sm, c, u, n, sm.zs);
        else
            unit_work<ES, false>(P, sm, c, u, n, zg);
    }
    tl_end(P.tl, TL_UNIT);
}

// hkv_step's S2-S4 for units too long to stage in one CTA, each split over a
// cluster of C CTAs: the same selection and PAD_MAX rows as k_unit. Units
// that reuse a rewrite, units short enough for one CTA, and units whose lists
// or cut bin outgrow shared memory are done by rank 0 alone, as k_unit does
// them (the other ranks then leave at once).
template <int ES, int C>
__global__ void __cluster_dims__(C, 1, 1) __launch_bounds__(NT, 1) k_unit_cluster(const __grid_constant__ Params P)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    USmem &sm = *reinterpret_cast<USmem *>(smem_raw);
    const Ctl c = make_ctl(P);
    const int u = blockIdx.x / C;
    const int rank = (int)cooperative_groups::this_cluster().block_rank();
    allow_dependents();
    wait_prior_grid();
    const int tb = rank == 0 ? TR_SEL + 16 * u : -1;
    HKV_TRACE_AT(tb);
    tl_start(P.tl, TL_UNIT);
    const int n = tier_len(P.sparse, u, c);
    const float *zg = P.z + (int64_t)u * P.z_stride;
    if (P.mti_left != nullptr && __ldcg(P.mti_left + u) > 0) {
        if (rank == 0)
            mti_reuse_outputs(P, c, u);  // the unit reuses its rewrite: nothing to select
    } else if (n <= ZSTAGE || cluster_chunk<C>(n) > ZSTAGE) {
        if (rank == 0) {
            if (n <= ZSTAGE) {
                unit_work<ES, true>(P, sm, c, u, n, sm.zs, zg);
            } else {
                const bool staged = stage_scores(zg, n, sm);
                if (staged)
                    unit_work<ES, true>(P, sm, c, u, n, sm.zs);
                else
                    unit_work<ES, false>(P, sm, c, u, n, zg);
            }
        }
    } else {
        // every rank reads the scorer's range words; rank 0 resets them for
        // the next step once the cluster is done with the unit
        if (threadIdx.x == 0) {
            const uint32_t kmax = __ldcg(P.urange + 2 * u), kmin = __ldcg(P.urange + 2 * u + 1);
            sm.redf[0] = kmax ? ord_val(kmax) : -INFINITY;
            sm.redf[1] = kmin ? ord_val(~kmin) : INFINITY;
        }
        __syncthreads();
        const float m = sm.redf[0], zlo = sm.redf[1];
        __syncthreads();
        HKV_TRACE_AT(tb < 0 ? -1 : tb + 4);
        const float beta = unit_beta(P, u, c), pu = unit_p(P, u, c);
        Selection s;
        const int st = select_compact_cluster<C>(zg, n, m, zlo, beta, pu, P.bmin, P.bmax, sm, s,
                                                 P.idx + (int64_t)u * P.bmax, P.bmax, tb, rank);
        if (rank == 0) {
            if (st != 0) {
                // the general path, alone (it reads and resets the range words)
                unit_work<ES, false>(P, sm, c, u, n, zg);
            } else {
                if (threadIdx.x == 0) {
                    P.sel_len[u] = s.k;
                    if (P.cut)
                        P.cut[u] = s.cut;
                    if (P.m_out)
                        P.m_out[u] = m;
                    if (P.logZ_out)
                        P.logZ_out[u] = (float)log(s.Z());
                    P.urange[2 * u] = 0;
                    P.urange[2 * u + 1] = 0;
                }
                HKV_TRACE_AT(tb + 5);
            }
        }
    }
    tl_end(P.tl, TL_UNIT);
}

// S2 standalone ([TS 2.B]) for unit u: m, logZ and optionally the calibrated
// probabilities. Z is summed exactly as the selection sums it (the 40-bit
// fixed-point weights, an exact integer sum), so m and logZ match hkv_step's
// bit for bit.
template <bool ZS>
__device__ __forceinline__ void calibrate_unit(const Params &P, USmem &sm, const Ctl &c, int u, int n,
                                               const float *zu)
{
    float m, zlo;
    unit_range<ZS>(zu, n, &m, &zlo, sm);
    const float bl2 = unit_beta(P, u, c) * LOG2E;
    unsigned long long part = 0;
    sweep_scores<ZS>(zu, n, [&](float z, int, bool valid) {
        if (valid)
            part += wfix(z, m, bl2);
    });
    const double Z = (double)block_sum_u64<NT>(part, sm.red) * (1.0 / 1099511627776.0);
    if (P.P_out != nullptr && n > 0) {
        const float inv = (float)(1.0 / Z);
        float *Pu = P.P_out + (int64_t)u * P.z_stride;
        sweep_scores<ZS>(zu, n, [&](float z, int j, bool valid) {
            if (valid)
                Pu[j] = wcal(z, m, bl2) * inv;
        });
    }
    if (threadIdx.x == 0) {
        P.m_out[u] = m;
        P.logZ_out[u] = n > 0 ? (float)log(Z) : -INFINITY;
    }
}

__global__ void __launch_bounds__(NT) k_calibrate(const __grid_constant__ Params P)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    USmem &sm = *reinterpret_cast<USmem *>(smem_raw);
    const Ctl c = make_ctl(P);
    const int u = blockIdx.x;
    const int n = tier_len(P.sparse, u, c);
    const float *zg = P.z + (int64_t)u * P.z_stride;
    if (stage_scores(zg, n, sm))
        calibrate_unit<true>(P, sm, c, u, n, sm.zs);
    else
        calibrate_unit<false>(P, sm, c, u, n, zg);
}

// Fitted temperature, one cluster of FIT_CTAS CTAs per unit: the target
// entropy from the scorer's per-head logit records (when P.logit is set; else
// P.h_target), then, when P.beta_out is set, the inverse temperature that
// meets it on the unit's scores P.z. The CTA of rank 0 writes the results.
template <int G>
__global__ void __cluster_dims__(FIT_CTAS, 1, 1) __launch_bounds__(NT, 1) k_fit(const __grid_constant__ Params P)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    FSmem &sm = *reinterpret_cast<FSmem *>(smem_raw);
    const Ctl c = make_ctl(P);
    const int u = blockIdx.x / FIT_CTAS;
    FitCluster cl;
    allow_dependents();
    wait_prior_grid();
    tl_start(P.tl, TL_FIT);
    const int n = tier_len(P.sparse, u, c);
    HKV_TRACE_IF(cl.rank == 0 && threadIdx.x == 0, TR_FIT + 16 * u);
    float target;
    if (P.logit != nullptr) {
        target = unit_attention_entropy<G>(P.logit + (int64_t)u * P.sparse.cap * logit_floats(G), n, sm, cl);
        if (P.h_out != nullptr && threadIdx.x == 0 && cl.rank == 0)
            P.h_out[u] = target;
    } else {
        target = __ldcg(P.h_target + u);
    }
    HKV_TRACE_IF(cl.rank == 0 && threadIdx.x == 0, TR_FIT + 16 * u + 1);
    if (P.beta_out != nullptr) {
        const float *zg = P.z + (int64_t)u * P.z_stride;
        const bool staged = stage_scores(zg, n, sm);
        HKV_TRACE_IF(cl.rank == 0 && threadIdx.x == 0, TR_FIT + 16 * u + 2);
        int evals = 0;
        const float beta = staged ? fit_unit<true>(sm.zs, n, target, sm, cl, c, &evals)
                                  : fit_unit<false>(zg, n, target, sm, cl, c, &evals);
        HKV_TRACE_IF(cl.rank == 0 && threadIdx.x == 0, TR_FIT + 16 * u + 3);
        if (cl.rank == 0)
            HKV_TRACE_VAL(TR_FIT + 16 * u + 4, evals);
        if (threadIdx.x == 0 && cl.rank == 0)
            P.beta_out[u] = beta;
    }
    // no CTA leaves while another may still read its shared memory
    cooperative_groups::this_cluster().sync();
    tl_end(P.tl, TL_FIT);
}

// FLAT_SUM rows and Rewrite Cache copies after the step's PAD_MAX compaction
// (one unit per CTA).
template <int ES>
__global__ void __launch_bounds__(NT) k_flatten(const __grid_constant__ Params P)
{
    __shared__ unsigned long long red[NT / 32];
    const Ctl c = make_ctl(P);
    const int u = blockIdx.x;
    wait_prior_grid();
    tl_start(P.tl, TL_FLAT);
    const int n = tier_len(P.sparse, u, c);
    const int k = max(0, min(__ldcg(P.sel_len + u), min(n, P.bmax)));
    const int32_t *src = P.idx + (int64_t)u * P.bmax;
    int64_t off = (int64_t)u * P.bmax;
    if (P.layout == HKV_LAYOUT_FLAT_SUM) {
        off = flat_offset(P, u, red);
        for (int i = threadIdx.x; i < k; i += NT)
            P.idx_user[off + i] = __ldcg(src + i);
        write_offsets(P, u, off);
    }
    if (P.k_out != nullptr)
        rewrite_rows(P, u, src, k, off, ES, c, n);
    tl_end(P.tl, TL_FLAT);
}

// =============================================================================
// Host side
// =============================================================================

std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_wait_ns{1000000000ull};
std::atomic<int32_t> g_withhold{0};
std::atomic<int32_t> g_timeline{0};

// Timeline words: the last 128 bytes of the workspace's 256-byte control area.
constexpr size_t TL_OFFSET = 128;

struct WsLayout {
    size_t ctl, urange, rec_range, part, idxbuf, zbuf, logits, total;
    int64_t z_stride;
    int part_slots;
};

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static int es_of(hkv_dtype d) { return d == HKV_BF16 ? 2 : 4; }

// The driver's tensor-map encoder, looked up once through the runtime
// (nullptr when the driver does not provide it).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// The sparse tier's K or V rows (rows_base: its k or v) as a 2-D tensor map
// for the attention's four-row gathers: every unit's cap rows one after
// another (row u cap + j), D elements a row, a box of one row. False (no map)
// unless the tier is laid out exactly that way: rows of D contiguous
// elements, units back to back.
static bool encode_rows_map(const hkv_problem *p, const hkv_tier *t, const void *rows_base, CUtensorMap *m)
{
    const auto enc = tensor_map_encoder();
    if (enc == nullptr || t == nullptr || rows_base == nullptr || t->cap <= 0)
        return false;
    const int64_t D = p->D;
    if (t->stride_t != D || t->stride_h != (int64_t)t->cap * D || t->stride_b != (int64_t)p->Hkv * t->cap * D)
        return false;
    const int64_t rows = (int64_t)p->B * p->Hkv * t->cap;
    if (rows >= (1ll << 31) || (reinterpret_cast<uintptr_t>(rows_base) & 15) != 0)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(D * es_of(p->dtype))};
    const cuuint32_t box[2] = {(cuuint32_t)D, 1};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, p->dtype == HKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
               const_cast<void *>(rows_base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The attention calls: both maps of the sparse tier, for four-row gathers of
// the selected tokens' K and V rows (neither when either cannot be made).
static void set_row_maps(const hkv_problem *p, const hkv_tier *sparse, Params &P)
{
    const bool ok = sparse != nullptr && encode_rows_map(p, sparse, sparse->k, &P.kmap) &&
                    encode_rows_map(p, sparse, sparse->v, &P.vmap);
    P.kmap_ok = ok ? 1 : 0;
    P.vmap_ok = ok ? 1 : 0;
}

static hkv_status check_tier(const hkv_tier *t, const hkv_problem *p, bool need_v)
{
    if (t == nullptr)
        return HKV_OK;
    const int es = es_of(p->dtype);
    if (t->cap < 0 || t->cap > (1 << 22))
        return HKV_ERR_INVALID_ARG;
    if (t->cap == 0)
        return HKV_OK;
    if (t->k == nullptr || t->len == nullptr || (need_v && t->v == nullptr))
        return HKV_ERR_INVALID_ARG;
    if (((uintptr_t)t->k & 15) || (t->v && ((uintptr_t)t->v & 15)))
        return HKV_ERR_INVALID_ARG;
    if (t->stride_t < p->D || t->stride_b < 0 || t->stride_h < 0)
        return HKV_ERR_INVALID_ARG;
    if ((t->stride_t * es) % 16 || (t->stride_h * es) % 16 || (t->stride_b * es) % 16)
        return HKV_ERR_INVALID_ARG;
    return HKV_OK;
}

static hkv_status check_problem(const hkv_problem *p)
{
    if (p == nullptr)
        return HKV_ERR_INVALID_ARG;
    if (p->B < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->Hq % p->Hkv != 0)
        return HKV_ERR_INVALID_ARG;
    if (p->dtype != HKV_BF16 && p->dtype != HKV_F32)
        return HKV_ERR_INVALID_ARG;
    if (p->bmin < 0 || p->bmax < p->bmin)
        return HKV_ERR_INVALID_ARG;
    if (p->layout != HKV_LAYOUT_PAD_MAX && p->layout != HKV_LAYOUT_FLAT_SUM)
        return HKV_ERR_INVALID_ARG;
    if (std::isnan(p->p) || !(p->scale >= 0.0f) || std::isinf(p->scale))
        return HKV_ERR_INVALID_ARG;
    if ((int64_t)p->B * p->Hkv > (1 << 24) || (int64_t)p->B * p->Hkv * (int64_t)p->bmax >= (1ll << 31))
        return HKV_ERR_INVALID_ARG;
    const int G = p->Hq / p->Hkv;
    if (p->D != 64 && p->D != 128)
        return HKV_ERR_UNSUPPORTED;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return HKV_ERR_UNSUPPORTED;
    return HKV_OK;
}

static int sm_count()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return sms;
}

// Streaming CTAs the attention records are sized for: one per SM of the
// current device (148 on B200, also assumed when no device can be queried).
static int stream_ctas()
{
    const int sms = sm_count();
    return sms > 0 ? sms : 148;
}

static WsLayout layout_of(const hkv_problem *p, const hkv_tier *dense, const hkv_tier *sparse,
                          const hkv_tier *cond)
{
    (void)dense;
    (void)cond;
    WsLayout L{};
    const int64_t units = (int64_t)p->B * p->Hkv;
    const int G = p->Hq / p->Hkv;
    const int ncap = sparse ? sparse->cap : 0;
    L.part_slots = (int)(2 * (stream_ctas() * (int64_t)AT_NW + units));
    L.z_stride = (int64_t)align_up((size_t)std::max(ncap, 1), 4);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes, 256);
        return at;
    };
    // what must start at zero comes first: status word, range words
    L.ctl = take(256);
    L.urange = take(units * 8);
    L.rec_range = take(units * 16);
    L.part = take((size_t)L.part_slots * part_stride(p->D, G) * 4);
    L.idxbuf = take(units * (size_t)std::max(p->bmax, 1) * 4);
    L.zbuf = take((size_t)units * L.z_stride * 4);
    L.logits = take((size_t)units * ncap * logit_floats(G) * 4);
    L.total = o;
    return L;
}

static Params base_params(const hkv_problem *p, const WsLayout &L, char *ws, const hkv_tier *dense,
                          const hkv_tier *sparse, const hkv_tier *cond)
{
    Params P{};
    P.B = p->B;
    P.Hq = p->Hq;
    P.Hkv = p->Hkv;
    P.D = p->D;
    P.G = p->Hq / p->Hkv;
    P.units = p->B * p->Hkv;
    P.scale = p->scale > 0.0f ? p->scale : 1.0f / std::sqrt((float)p->D);
    P.p = p->p;
    P.bmin = p->bmin;
    P.bmax = p->bmax;
    P.layout = p->layout;
    P.inv_temp = p->inv_temp;
    P.p_unit = p->p_unit;
    P.z_stride = L.z_stride;
    P.wait_ns = g_wait_ns.load();
    P.withhold = g_withhold.load();
    P.ctl = reinterpret_cast<uint32_t *>(ws + L.ctl);
    P.tl = g_timeline.load() ? reinterpret_cast<unsigned long long *>(ws + L.ctl + TL_OFFSET) : nullptr;
    P.rec_range = reinterpret_cast<int32_t *>(ws + L.rec_range);
    P.part = reinterpret_cast<float *>(ws + L.part);
    P.part_slots = L.part_slots;
    // lines laid out by actual counts when the counts fit shared memory and
    // every line position fits 31 bits
    const int64_t span = (int64_t)(dense ? dense->cap : 0) + std::min(p->bmax, sparse ? sparse->cap : 0) +
                         (cond ? cond->cap : 0);
    P.attn_prefix = P.units <= PREFIX_CAP && (int64_t)P.units * span < (1ll << 31);
    P.unit_ctas = P.units;
    return P;
}

static TierP tier_p(const hkv_tier *t)
{
    TierP r{};
    if (t == nullptr || t->cap == 0)
        return r;
    r.k = static_cast<const char *>(t->k);
    r.v = static_cast<const char *>(t->v);
    r.sb = t->stride_b;
    r.sh = t->stride_h;
    r.st = t->stride_t;
    r.cap = t->cap;
    r.len = t->len;
    return r;
}

static hkv_status check_ws(void *ws, size_t ws_bytes, const WsLayout &L)
{
    if (ws == nullptr || ((uintptr_t)ws & 255) || ws_bytes < L.total)
        return HKV_ERR_WORKSPACE;
    return HKV_OK;
}

// Per-device cache of kernel attributes (dynamic shared memory opt-in and
// resident CTAs per SM).
struct KernelInfo {
    const void *fn;
    int device;
    int blocks_per_sm;
};
static std::mutex g_mu;
static KernelInfo g_info[256];
static int g_ninfo = 0;

static hkv_status prepare(const void *fn, int threads, size_t smem, int *blocks_per_sm)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return HKV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_ninfo; ++i)
        if (g_info[i].fn == fn && g_info[i].device == dev) {
            if (blocks_per_sm)
                *blocks_per_sm = g_info[i].blocks_per_sm;
            return HKV_OK;
        }
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return HKV_ERR_CUDA;
    int bps = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, fn, threads, smem) != cudaSuccess)
        return HKV_ERR_CUDA;
    if (g_ninfo < 256)
        g_info[g_ninfo++] = KernelInfo{fn, dev, bps};
    if (blocks_per_sm)
        *blocks_per_sm = bps;
    return HKV_OK;
}

// Launch `kernel` over `grid` CTAs. With pdl the launch is a programmatic
// dependent of the previous kernel on the stream: it may start early, and the
// kernel calls wait_prior_grid() before it reads that kernel's results.
template <typename K>
static hkv_status launch(K kernel, int grid, int threads, size_t smem, cudaStream_t stream, const Params &P,
                         bool pdl)
{
    if (grid <= 0)
        return HKV_OK;
    hkv_status s = prepare((const void *)kernel, threads, smem, nullptr);
    if (s != HKV_OK)
        return s;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kernel, P) != cudaSuccess)
        return HKV_ERR_CUDA;
    g_launches.fetch_add(1);
    return HKV_OK;
}

// Streaming kernels: as many CTAs as are resident at once (one per SM), at
// most max_ctas.
template <typename K>
static hkv_status launch_stream(K kernel, int threads, size_t smem, int max_ctas, cudaStream_t stream,
                                const Params &P, bool pdl)
{
    int bps = 0;
    hkv_status s = prepare((const void *)kernel, threads, smem, &bps);
    if (s != HKV_OK)
        return s;
    const int sms = sm_count();
    if (sms <= 0 || bps <= 0)
        return HKV_ERR_CUDA;
    return launch(kernel, std::max(1, std::min(max_ctas, bps * sms)), threads, smem, stream, P, pdl);
}

// Dispatch over the compile-time (element size, head dim, group size).
template <template <int, int, int> class F, typename... A>
static hkv_status dispatch(const hkv_problem *p, A &&...args)
{
    const int es = es_of(p->dtype), G = p->Hq / p->Hkv, D = p->D;
#define HKV_CASE(E, DD, GG) \
    if (es == E && D == DD && G == GG) \
        return F<E, DD, GG>::run(args...);
#define HKV_GCASES(E, DD) HKV_CASE(E, DD, 1) HKV_CASE(E, DD, 2) HKV_CASE(E, DD, 4) HKV_CASE(E, DD, 8)
    HKV_GCASES(2, 128)
    HKV_GCASES(2, 64)
    HKV_GCASES(4, 128)
    HKV_GCASES(4, 64)
#undef HKV_GCASES
#undef HKV_CASE
    return HKV_ERR_UNSUPPORTED;
}

template <int ES, int D, int G>
struct RunScore {
    static hkv_status run(const Params &P, cudaStream_t s, bool pdl)
    {
        return launch_stream(k_score_stream<ES, D, G>, sc_nw(G) * 32, sizeof(typename ScoreJob<ES, D, G>::Smem),
                             1 << 20, s, P, pdl);
    }
};

template <int ES, int D, int G>
struct RunAttn {
    // attention then merge
    static hkv_status run(const Params &P, cudaStream_t s, bool pdl)
    {
        // the records hold 2 x (CTAs x warps + units) slots
        const int max_ctas = (P.part_slots / 2 - P.units) / AT_NW;
        if (max_ctas < 1)
            return HKV_ERR_WORKSPACE;
        // with fewer units than SMs, line A goes to the CTAs that start while
        // the selection kernel (one CTA per unit) runs
        const int sms = sm_count();
        Params Q = P;
        Q.attn_a_ctas = (pdl && P.unit_ctas < sms) ? sms - P.unit_ctas : (1 << 30);
        hkv_status st = launch_stream(k_attn_stream<ES, D, G>, AT_NW * 32, sizeof(AttnSmem<ES, D, G>), max_ctas, s,
                                      Q, pdl);
        if (st != HKV_OK)
            return st;
        return launch(k_merge<D, G>, P.units, MERGE_WARPS * 32, 0, s, P, true);
    }
};

template <int ES, int D, int G>
struct RunFit {
    static hkv_status run(const Params &P, cudaStream_t s, bool pdl)
    {
        return launch(k_fit<G>, P.units * FIT_CTAS, NT, sizeof(FSmem), s, P, pdl);  // clusters of FIT_CTAS
    }
};

// split: CTAs per unit (1, 2 or 4)
static hkv_status launch_unit(const hkv_problem *prob, const Params &P, cudaStream_t s, bool pdl, int split = 1)
{
    const bool bf = prob->dtype == HKV_BF16;
    if (split == 4)
        return bf ? launch(k_unit_cluster<2, 4>, 4 * P.units, NT, sizeof(USmem), s, P, pdl)
                  : launch(k_unit_cluster<4, 4>, 4 * P.units, NT, sizeof(USmem), s, P, pdl);
    if (split == 2)
        return bf ? launch(k_unit_cluster<2, 2>, 2 * P.units, NT, sizeof(USmem), s, P, pdl)
                  : launch(k_unit_cluster<4, 2>, 2 * P.units, NT, sizeof(USmem), s, P, pdl);
    if (prob->dtype == HKV_BF16)
        return launch(k_unit<2>, P.units, NT, sizeof(USmem), s, P, pdl);
    return launch(k_unit<4>, P.units, NT, sizeof(USmem), s, P, pdl);
}

}  // namespace hkv

using namespace hkv;

namespace {

// Common validation of a compute call; fills the layout and the parameters.
hkv_status prologue(const hkv_problem *prob, const hkv_tier *dense, const hkv_tier *sparse, const hkv_tier *cond,
                    bool need_v, void *ws, size_t ws_bytes, WsLayout *L, Params *P)
{
    hkv_status s = check_problem(prob);
    if (s != HKV_OK)
        return s;
    if ((s = check_tier(dense, prob, true)) != HKV_OK || (s = check_tier(sparse, prob, need_v)) != HKV_OK ||
        (s = check_tier(cond, prob, true)) != HKV_OK)
        return s;
    *L = layout_of(prob, dense, sparse, cond);
    if ((s = check_ws(ws, ws_bytes, *L)) != HKV_OK)
        return s;
    *P = base_params(prob, *L, static_cast<char *>(ws), dense, sparse, cond);
    P->dense = tier_p(dense);
    P->sparse = tier_p(sparse);
    P->cond = tier_p(cond);
    return HKV_OK;
}

bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

}  // namespace

namespace hkv {

// ---- Rewrite Cache vs Sparse Loading ([TS 2.C] Trade-off Management) --------
//
// After the step's attention, per unit: a unit that reused its rewrite counts
// one step down; any other unit (it was scored and selected) takes the trigger
// on its fresh budget k -- Rewrite Cache when k > L_upper, Sparse Loading when
// k < L_lower, the previous mode in between -- and under Rewrite Cache copies
// its k selected K and V rows into the rewrite buffer, which then serves
// H(k) = max(1, floor(mti_cap / k)) steps in all (this one included): a
// rewrite of k rows kept H steps holds k H <= mti_cap row-steps of memory.
// A cluster of MTI_CTAS CTAs per unit splits the rows; they meet once, before
// the unit's state (read by all of them) is updated.

constexpr int MTI_CTAS = 4;
constexpr int MTI_NT = 256;
constexpr int MTI_BATCH = 8;  // rewrite copy: 16-byte chunks a thread has in flight

struct MtiP {
    const char *sk, *sv;                   // sparse tier
    int64_t ssb, ssh, sst;                 // byte strides
    char *rk, *rv;                         // rewrite buffer
    int64_t rsb, rsh, rst;
    const int32_t *idx, *sel_len, *slen;   // the step's PAD_MAX rows and budgets; sparse lengths
    int32_t *mode, *left, *rw_len, *rw_idx;
    int32_t Hkv, bmax, rowb, ncap, L_lower, L_upper;
    int64_t mti_cap;
    uint32_t *status;
    unsigned long long *tl;
};

__global__ void __cluster_dims__(MTI_CTAS, 1, 1) __launch_bounds__(MTI_NT) k_mti(const __grid_constant__ MtiP M)
{
    auto cluster = cooperative_groups::this_cluster();
    const int r = (int)cluster.block_rank();
    const int u = blockIdx.x / MTI_CTAS;
    wait_prior_grid();  // the step's attention has read the state and the buffer
    tl_start(M.tl, TL_MTI);
    const int left0 = __ldcg(M.left + u);
    if (left0 > 0) {  // reused this step
        cluster.sync();
        if (r == 0 && threadIdx.x == 0)
            M.left[u] = left0 - 1;
        tl_end(M.tl, TL_MTI);
        return;
    }
    const int k = max(0, min(__ldcg(M.sel_len + u), M.bmax));
    const int mode0 = __ldcg(M.mode + u);
    const int mode1 = k > M.L_upper ? 1 : (k < M.L_lower ? 0 : (mode0 != 0 ? 1 : 0));
    if (mode1) {
        // rows [k r / MTI_CTAS, k (r + 1) / MTI_CTAS) of the selection, in 16-byte chunks
        const int b = u / M.Hkv, h = u - b * M.Hkv;
        const int n = max(0, min(__ldcg(M.slen + u), M.ncap));
        const int i0 = k * r / MTI_CTAS, i1 = k * (r + 1) / MTI_CTAS;
        const int ch = M.rowb / 16;
        const int32_t *row = M.idx + (int64_t)u * M.bmax;
        // MTI_BATCH chunks a thread, all loads in flight before the stores
        const int total = (i1 - i0) * 2 * ch;
        for (int x0 = threadIdx.x; x0 < total; x0 += MTI_NT * MTI_BATCH) {
            uint4 val[MTI_BATCH];
            char *dst[MTI_BATCH];
#pragma unroll
            for (int e = 0; e < MTI_BATCH; ++e) {
                const int x = x0 + e * MTI_NT;
                dst[e] = nullptr;
                if (x >= total)
                    continue;
                const int i = i0 + x / (2 * ch), q = x % (2 * ch);
                const bool isk = q < ch;
                const int j0 = __ldcg(row + i);
                int j = j0;
                if (j < 0 || j >= n) {
                    atomicOr(M.status, HKV_DEV_BAD_INDEX);
                    j = 0;
                }
                const char *src = (isk ? M.sk : M.sv) + (int64_t)b * M.ssb + (int64_t)h * M.ssh + (int64_t)j * M.sst;
                const int off = (isk ? q : q - ch) * 16;
                val[e] = __ldcs(reinterpret_cast<const uint4 *>(src + off));
                dst[e] = (isk ? M.rk : M.rv) + (int64_t)b * M.rsb + (int64_t)h * M.rsh + (int64_t)i * M.rst + off;
                if (q == 0)
                    M.rw_idx[(int64_t)u * M.bmax + i] = j0;
            }
#pragma unroll
            for (int e = 0; e < MTI_BATCH; ++e)
                if (dst[e] != nullptr)
                    *reinterpret_cast<uint4 *>(dst[e]) = val[e];
        }
    }
    cluster.sync();
    if (r == 0 && threadIdx.x == 0) {
        M.mode[u] = mode1;
        if (mode1) {
            const int64_t H = k > 0 ? max((int64_t)1, min(M.mti_cap / k, (int64_t)1 << 30)) : 1;
            M.rw_len[u] = k;
            M.left[u] = (int32_t)(H - 1);
        } else {
            M.rw_len[u] = 0;
            M.left[u] = 0;
        }
    }
    tl_end(M.tl, TL_MTI);
}

}  // namespace hkv

namespace {

// The decode step (hkv_step), and with `mti` the step under the Rewrite Cache /
// Sparse Loading trigger (hkv_step_mti).
hkv_status step_impl(const hkv_problem *prob, const void *q, const hkv_tier *dense, const hkv_tier *sparse,
                     const hkv_tier *condensed, const hkv_step_out *o, const hkv_mti *mti, void *ws, size_t ws_bytes,
                     hkv_stream_t stream)
{
    WsLayout L;
    Params P;
    if (sparse == nullptr || o == nullptr)
        return HKV_ERR_INVALID_ARG;
    hkv_status s = prologue(prob, dense, sparse, condensed, true, ws, ws_bytes, &L, &P);
    if (s != HKV_OK)
        return s;
    if (q == nullptr || !aligned(q, 16) || o->out == nullptr || o->sel_len == nullptr || o->idx == nullptr)
        return HKV_ERR_INVALID_ARG;
    const bool flat = prob->layout == HKV_LAYOUT_FLAT_SUM;
    if (flat && o->offsets == nullptr)
        return HKV_ERR_INVALID_ARG;
    const bool rewrite = o->k_out != nullptr || o->v_out != nullptr;
    if (rewrite && (o->k_out == nullptr || o->v_out == nullptr || !aligned(o->k_out, 16) || !aligned(o->v_out, 16)))
        return HKV_ERR_INVALID_ARG;
    if (o->z && !aligned(o->z, 4))
        return HKV_ERR_INVALID_ARG;
    if ((o->h_attn != nullptr && o->beta_fit == nullptr) || (o->beta_fit && !aligned(o->beta_fit, 4)) ||
        (o->h_attn && !aligned(o->h_attn, 4)))
        return HKV_ERR_INVALID_ARG;
    if (mti != nullptr) {
        // the rewrite buffer is the Rewrite Cache here; a fitted temperature
        // would need the scores that reusing units skip
        if (rewrite || o->beta_fit != nullptr)
            return HKV_ERR_INVALID_ARG;
        if (mti->L_lower < 0 || mti->L_upper < mti->L_lower || mti->mti_cap < 0 || mti->mode == nullptr ||
            mti->left == nullptr || mti->rw_idx == nullptr || !aligned(mti->mode, 4) || !aligned(mti->left, 4) ||
            !aligned(mti->rw_idx, 4))
            return HKV_ERR_INVALID_ARG;
        if ((s = check_tier(&mti->rewrite, prob, true)) != HKV_OK)
            return s;
        if (mti->rewrite.cap < prob->bmax || (prob->bmax > 0 && mti->rewrite.len == nullptr))
            return HKV_ERR_INVALID_ARG;
        // units and lines small enough for the attention's exact (prefix) layout
        const int64_t span = (int64_t)(dense ? dense->cap : 0) + mti->rewrite.cap + (condensed ? condensed->cap : 0) +
                             std::min(prob->bmax, sparse->cap);
        if ((int64_t)P.units > PREFIX_CAP || (int64_t)P.units * span >= (1ll << 31))
            return HKV_ERR_UNSUPPORTED;
    }
    if (P.units == 0)
        return HKV_OK;
    char *wsb = static_cast<char *>(ws);
    const cudaStream_t st = (cudaStream_t)stream;
    P.q = static_cast<const char *>(q);
    P.z = o->z ? o->z : reinterpret_cast<float *>(wsb + L.zbuf);
    P.z_stride = o->z ? sparse->cap : L.z_stride;
    P.sel_len = o->sel_len;
    P.cut = o->cut;
    P.idx = flat ? reinterpret_cast<int32_t *>(wsb + L.idxbuf) : o->idx;  // PAD_MAX rows for the attention
    P.idx_user = o->idx;
    P.offsets = o->offsets;
    P.out = o->out;
    P.lse = o->lse;
    P.m_out = o->m;
    P.logZ_out = o->logZ;
    P.k_out = static_cast<char *>(o->k_out);
    P.v_out = static_cast<char *>(o->v_out);
    P.logit = reinterpret_cast<float *>(wsb + L.logits);  // scorer -> attention of the selected tokens
    P.vmap_ok = encode_rows_map(prob, sparse, sparse->v, &P.vmap) ? 1 : 0;  // four-row gathers of selected V rows
    P.layout = HKV_LAYOUT_PAD_MAX;  // the three kernels work on PAD_MAX rows
    if (mti != nullptr) {
        P.mti_left = mti->left;
        P.rw = tier_p(&mti->rewrite);
        P.rw_idx = mti->rw_idx;
        P.attn_prefix = 1;
    }
    // 1. scores, and the score range of each unit (launched in stream order:
    // as a programmatic dependent of the previous step its CTAs would sit on
    // SMs the previous attention is leaving, which measured slower)
    const bool scored = sparse->cap > 0;
    Params S = P;
    S.urange = reinterpret_cast<uint32_t *>(wsb + L.urange);
    // the scorer waits for the previous kernel before reading anything; PDL
    // only hides its launch behind that kernel's tail
    if (scored && (s = dispatch<RunScore>(prob, S, st, true)) != HKV_OK)
        return s;
    // 1b. optionally the fitted inverse temperature of every unit, from the
    // scorer's logit records and scores; the selection then uses it
    Params U = S;
    if (o->beta_fit != nullptr) {
        Params F = S;
        F.urange = nullptr;
        F.beta_out = o->beta_fit;
        F.h_out = o->h_attn;
        if ((s = dispatch<RunFit>(prob, F, st, scored)) != HKV_OK)
            return s;
        U.inv_temp = o->beta_fit;
    }
    // 2. calibration, Top-p budget, cut and compaction, per unit
    U.have_range = scored;
    U.do_select = 1;
    U.do_compact = 1;
    // units longer than one CTA can stage are split over a cluster of CTAs
    // (one CTA would sweep such a unit from L2 several times): four when all
    // the clusters fit the SMs at once, else two when two CTAs can stage it
    int split = 1;
    if (scored && sparse->cap > ZSTAGE) {
        if (4 * P.units <= sm_count() && cluster_chunk<4>(sparse->cap) <= ZSTAGE)
            split = 4;
        else if (cluster_chunk<2>(sparse->cap) <= ZSTAGE)
            split = 2;
    }
    if ((s = launch_unit(prob, U, st, true, split)) != HKV_OK)
        return s;
    P.unit_ctas = split * P.units;
    // 3. attention over the three tiers and the merge of each unit
    if ((s = dispatch<RunAttn>(prob, P, st, true)) != HKV_OK)
        return s;
    if (flat || rewrite) {
        P.layout = prob->layout;
        s = prob->dtype == HKV_BF16 ? launch(k_flatten<2>, P.units, NT, 0, st, P, true)
                                    : launch(k_flatten<4>, P.units, NT, 0, st, P, true);
        if (s != HKV_OK)
            return s;
    }
    if (mti == nullptr)
        return HKV_OK;
    // 4. the trigger, and the rewrites it asks for
    const int es = es_of(prob->dtype);
    MtiP M{};
    M.sk = static_cast<const char *>(sparse->k);
    M.sv = static_cast<const char *>(sparse->v);
    M.ssb = sparse->stride_b * es;
    M.ssh = sparse->stride_h * es;
    M.sst = sparse->stride_t * es;
    M.rk = static_cast<char *>(const_cast<void *>(mti->rewrite.k));
    M.rv = static_cast<char *>(const_cast<void *>(mti->rewrite.v));
    M.rsb = mti->rewrite.stride_b * es;
    M.rsh = mti->rewrite.stride_h * es;
    M.rst = mti->rewrite.stride_t * es;
    M.idx = P.idx;
    M.sel_len = o->sel_len;
    M.slen = sparse->len;
    M.mode = mti->mode;
    M.left = mti->left;
    M.rw_len = const_cast<int32_t *>(mti->rewrite.len);
    M.rw_idx = mti->rw_idx;
    M.Hkv = prob->Hkv;
    M.bmax = prob->bmax;
    M.rowb = prob->D * es;
    M.ncap = sparse->cap;
    M.L_lower = mti->L_lower;
    M.L_upper = mti->L_upper;
    M.mti_cap = mti->mti_cap;
    M.status = P.ctl;
    M.tl = P.tl;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(P.units * MTI_CTAS));
    cfg.blockDim = dim3(MTI_NT);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_mti, M) != cudaSuccess)
        return HKV_ERR_CUDA;
    g_launches.fetch_add(1);
    return HKV_OK;
}

}  // namespace

extern "C" {

const char *hkv_status_string(hkv_status s)
{
    switch (s) {
    case HKV_OK: return "HKV_OK";
    case HKV_ERR_INVALID_ARG: return "HKV_ERR_INVALID_ARG";
    case HKV_ERR_UNSUPPORTED: return "HKV_ERR_UNSUPPORTED";
    case HKV_ERR_CUDA: return "HKV_ERR_CUDA";
    case HKV_ERR_TIMEOUT: return "HKV_ERR_TIMEOUT";
    case HKV_ERR_DEVICE: return "HKV_ERR_DEVICE";
    case HKV_ERR_WORKSPACE: return "HKV_ERR_WORKSPACE";
    }
    return "HKV_ERR_UNKNOWN";
}

uint64_t hkv_launch_count(void) { return g_launches.load(); }

hkv_status hkv_set_wait_limit_ns(uint64_t ns)
{
    if (ns == 0)
        return HKV_ERR_INVALID_ARG;
    g_wait_ns.store(ns);
    return HKV_OK;
}

hkv_status hkv_set_timeline(int32_t on)
{
    g_timeline.store(on ? 1 : 0);
    return HKV_OK;
}

hkv_status hkv_read_timeline(void *ws, uint64_t *start_end, hkv_stream_t stream)
{
    if (ws == nullptr || ((uintptr_t)ws & 255))
        return HKV_ERR_WORKSPACE;
    if (start_end == nullptr)
        return HKV_ERR_INVALID_ARG;
    unsigned long long w[16];
    cudaStream_t s = (cudaStream_t)stream;
    char *tl = static_cast<char *>(ws) + TL_OFFSET;
    if (cudaMemcpyAsync(w, tl, sizeof w, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess || cudaMemsetAsync(tl, 0, sizeof w, s) != cudaSuccess)
        return HKV_ERR_CUDA;
    for (int k = 0; k < HKV_TL_KINDS; ++k) {
        start_end[2 * k] = w[k] ? ~w[k] : 0;
        start_end[2 * k + 1] = w[8 + k];
    }
    return HKV_OK;
}

hkv_status hkv_debug_withhold_publish(int32_t on)
{
    g_withhold.store(on ? 1 : 0);
    return HKV_OK;
}

hkv_status hkv_workspace_size(const hkv_problem *prob, const hkv_tier *dense, const hkv_tier *sparse,
                              const hkv_tier *condensed, size_t *bytes)
{
    hkv_status s = check_problem(prob);
    if (s != HKV_OK)
        return s;
    if (bytes == nullptr)
        return HKV_ERR_INVALID_ARG;
    if ((s = check_tier(dense, prob, true)) || (s = check_tier(sparse, prob, false)) ||
        (s = check_tier(condensed, prob, true)))
        return s;
    *bytes = layout_of(prob, dense, sparse, condensed).total;
    return HKV_OK;
}

hkv_status hkv_workspace_init(void *ws, size_t bytes, hkv_stream_t stream)
{
    if (ws == nullptr || bytes < 256)
        return HKV_ERR_WORKSPACE;
    return cudaMemsetAsync(ws, 0, bytes, (cudaStream_t)stream) == cudaSuccess ? HKV_OK : HKV_ERR_CUDA;
}

hkv_status hkv_get_status(void *ws, uint32_t *flags, hkv_stream_t stream)
{
    if (ws == nullptr)
        return HKV_ERR_WORKSPACE;
    uint32_t word = 0;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&word, ws, sizeof word, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess || cudaMemsetAsync(ws, 0, sizeof word, s) != cudaSuccess)
        return HKV_ERR_CUDA;
    if (flags)
        *flags = word;
    if (word == 0)
        return HKV_OK;
    return (word & HKV_DEV_TIMEOUT) ? HKV_ERR_TIMEOUT : HKV_ERR_DEVICE;
}

hkv_status hkv_score(const hkv_problem *prob, const void *q, const hkv_tier *sparse, float *z, int64_t z_stride,
                     void *ws, size_t ws_bytes, hkv_stream_t stream)
{
    WsLayout L;
    Params P;
    if (sparse == nullptr)
        return HKV_ERR_INVALID_ARG;
    hkv_status s = prologue(prob, nullptr, sparse, nullptr, false, ws, ws_bytes, &L, &P);
    if (s != HKV_OK)
        return s;
    if (q == nullptr || !aligned(q, 16) || z == nullptr || !aligned(z, 4) || z_stride < sparse->cap)
        return HKV_ERR_INVALID_ARG;
    if (P.units == 0 || sparse->cap == 0)
        return HKV_OK;
    P.q = static_cast<const char *>(q);
    P.z = z;
    P.z_stride = z_stride;
    return dispatch<RunScore>(prob, P, (cudaStream_t)stream, false);
}

hkv_status hkv_calibrate(const hkv_problem *prob, const float *z, int64_t z_stride, const hkv_tier *sparse,
                         float *Pout, float *m, float *logZ, void *ws, size_t ws_bytes, hkv_stream_t stream)
{
    WsLayout L;
    Params P;
    if (sparse == nullptr)
        return HKV_ERR_INVALID_ARG;
    hkv_status s = prologue(prob, nullptr, sparse, nullptr, false, ws, ws_bytes, &L, &P);
    if (s != HKV_OK)
        return s;
    if (z == nullptr || !aligned(z, 4) || z_stride < sparse->cap || m == nullptr || logZ == nullptr ||
        (Pout && !aligned(Pout, 4)))
        return HKV_ERR_INVALID_ARG;
    P.z = const_cast<float *>(z);
    P.z_stride = z_stride;
    P.P_out = Pout;
    P.m_out = m;
    P.logZ_out = logZ;
    return launch(k_calibrate, P.units, NT, sizeof(USmem), (cudaStream_t)stream, P, false);
}

hkv_status hkv_topp_select(const hkv_problem *prob, const float *z, int64_t z_stride, const hkv_tier *sparse,
                           int32_t *sel_len, hkv_cut *cut, void *ws, size_t ws_bytes, hkv_stream_t stream)
{
    WsLayout L;
    Params P;
    if (sparse == nullptr)
        return HKV_ERR_INVALID_ARG;
    hkv_status s = prologue(prob, nullptr, sparse, nullptr, false, ws, ws_bytes, &L, &P);
    if (s != HKV_OK)
        return s;
    if (z == nullptr || !aligned(z, 4) || z_stride < sparse->cap || sel_len == nullptr || cut == nullptr)
        return HKV_ERR_INVALID_ARG;
    P.z = const_cast<float *>(z);
    P.z_stride = z_stride;
    P.sel_len = sel_len;
    P.cut = cut;
    P.do_select = 1;
    return launch_unit(prob, P, (cudaStream_t)stream, false);
}

hkv_status hkv_compact(const hkv_problem *prob, const float *z, int64_t z_stride, const hkv_tier *sparse,
                       const int32_t *sel_len, const hkv_cut *cut, int32_t *idx, int32_t *offsets, void *k_out,
                       void *v_out, void *ws, size_t ws_bytes, hkv_stream_t stream)
{
    WsLayout L;
    Params P;
    if (sparse == nullptr)
        return HKV_ERR_INVALID_ARG;
    const bool rewrite = k_out != nullptr || v_out != nullptr;
    hkv_status s = prologue(prob, nullptr, sparse, nullptr, rewrite, ws, ws_bytes, &L, &P);
    if (s != HKV_OK)
        return s;
    if (z == nullptr || !aligned(z, 4) || z_stride < sparse->cap || sel_len == nullptr || cut == nullptr ||
        idx == nullptr)
        return HKV_ERR_INVALID_ARG;
    if (prob->layout == HKV_LAYOUT_FLAT_SUM && offsets == nullptr)
        return HKV_ERR_INVALID_ARG;
    if (rewrite && (k_out == nullptr || v_out == nullptr || !aligned(k_out, 16) || !aligned(v_out, 16) ||
                    sparse->cap == 0))
        return HKV_ERR_INVALID_ARG;
    P.z = const_cast<float *>(z);
    P.z_stride = z_stride;
    P.sel_len = const_cast<int32_t *>(sel_len);
    P.cut = const_cast<hkv_cut *>(cut);
    P.idx = idx;
    P.offsets = offsets;
    P.k_out = static_cast<char *>(k_out);
    P.v_out = static_cast<char *>(v_out);
    P.do_compact = 1;
    return launch_unit(prob, P, (cudaStream_t)stream, false);
}

hkv_status hkv_cascade_decode(const hkv_problem *prob, const void *q, const hkv_tier *dense,
                              const hkv_tier *sparse, const int32_t *idx, const int32_t *offsets,
                              const int32_t *sel_len, const hkv_tier *condensed, float *out, float *lse, void *ws,
                              size_t ws_bytes, hkv_stream_t stream)
{
    WsLayout L;
    Params P;
    hkv_status s = prologue(prob, dense, sparse, condensed, true, ws, ws_bytes, &L, &P);
    if (s != HKV_OK)
        return s;
    if (q == nullptr || !aligned(q, 16) || out == nullptr)
        return HKV_ERR_INVALID_ARG;
    if (sparse != nullptr && sparse->cap > 0) {
        if (idx == nullptr || sel_len == nullptr)
            return HKV_ERR_INVALID_ARG;
        if (prob->layout == HKV_LAYOUT_FLAT_SUM && offsets == nullptr)
            return HKV_ERR_INVALID_ARG;
    }
    if (P.units == 0)
        return HKV_OK;
    P.q = static_cast<const char *>(q);
    P.idx = const_cast<int32_t *>(idx);
    P.offsets = const_cast<int32_t *>(offsets);
    P.sel_len = const_cast<int32_t *>(sel_len);
    P.out = out;
    P.lse = lse;
    set_row_maps(prob, sparse, P);
    return dispatch<RunAttn>(prob, P, (cudaStream_t)stream, false);
}

hkv_status hkv_step(const hkv_problem *prob, const void *q, const hkv_tier *dense, const hkv_tier *sparse,
                    const hkv_tier *condensed, const hkv_step_out *o, void *ws, size_t ws_bytes,
                    hkv_stream_t stream)
{
    return step_impl(prob, q, dense, sparse, condensed, o, nullptr, ws, ws_bytes, stream);
}

hkv_status hkv_step_mti(const hkv_problem *prob, const void *q, const hkv_tier *dense, const hkv_tier *sparse,
                        const hkv_tier *condensed, const hkv_mti *mti, const hkv_step_out *o, void *ws,
                        size_t ws_bytes, hkv_stream_t stream)
{
    if (mti == nullptr)
        return HKV_ERR_INVALID_ARG;
    return step_impl(prob, q, dense, sparse, condensed, o, mti, ws, ws_bytes, stream);
}

hkv_status hkv_attention_entropy(const hkv_problem *prob, const void *q, const hkv_tier *sparse, float *h, void *ws,
                                 size_t ws_bytes, hkv_stream_t stream)
{
    WsLayout L;
    Params P;
    if (sparse == nullptr)
        return HKV_ERR_INVALID_ARG;
    hkv_status s = prologue(prob, nullptr, sparse, nullptr, false, ws, ws_bytes, &L, &P);
    if (s != HKV_OK)
        return s;
    if (q == nullptr || !aligned(q, 16) || h == nullptr || !aligned(h, 4))
        return HKV_ERR_INVALID_ARG;
    if (P.units == 0)
        return HKV_OK;
    char *wsb = static_cast<char *>(ws);
    const cudaStream_t st = (cudaStream_t)stream;
    P.q = static_cast<const char *>(q);
    P.z = reinterpret_cast<float *>(wsb + L.zbuf);
    P.z_stride = L.z_stride;
    P.logit = reinterpret_cast<float *>(wsb + L.logits);
    const bool scored = sparse->cap > 0;
    if (scored && (s = dispatch<RunScore>(prob, P, st, false)) != HKV_OK)
        return s;
    P.h_out = h;
    return dispatch<RunFit>(prob, P, st, scored);
}

hkv_status hkv_fit_temperature(const hkv_problem *prob, const float *z, int64_t z_stride, const hkv_tier *sparse,
                               const float *h_target, float *beta, void *ws, size_t ws_bytes, hkv_stream_t stream)
{
    WsLayout L;
    Params P;
    if (sparse == nullptr)
        return HKV_ERR_INVALID_ARG;
    hkv_status s = prologue(prob, nullptr, sparse, nullptr, false, ws, ws_bytes, &L, &P);
    if (s != HKV_OK)
        return s;
    if (h_target == nullptr || !aligned(h_target, 4) || beta == nullptr || !aligned(beta, 4))
        return HKV_ERR_INVALID_ARG;
    if (sparse->cap > 0 && (z == nullptr || !aligned(z, 4) || z_stride < sparse->cap))
        return HKV_ERR_INVALID_ARG;
    if (P.units == 0)
        return HKV_OK;
    P.z = const_cast<float *>(z);
    P.z_stride = z_stride;
    P.h_target = h_target;
    P.beta_out = beta;
    return dispatch<RunFit>(prob, P, (cudaStream_t)stream, false);
}

}  // extern "C"

// =============================================================================
// No-allocation cascade decode
//
// For callers that cannot allocate device memory where they decode (an engine
// that gives nearly all HBM to its KV pool up front and forbids allocation on
// the decode path, or a plugin hook with no workspace to hand over). The
// kernel and its arguments are those of hkv_cascade_decode; only the scratch
// moves from the caller's workspace into a fixed array of this library.
// =============================================================================

namespace hkv {

// The scratch, one copy per device that loads the library. In host code this
// name is only a stand-in for the symbol, never a device address: kernels get
// the address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[HKV_NOALLOC_SCRATCH_BYTES];

constexpr int NOALLOC_MAX_DEVICES = 64;
static std::mutex g_noalloc_mu;
static void *g_noalloc_ptr[NOALLOC_MAX_DEVICES];

// Device address of the scratch in the current device's context. A call made
// outside stream capture looks it up afresh (cudaGetSymbolAddress, which also
// loads the module on first use), so an address never outlives the context
// it belongs to (a cudaDeviceReset, another primary context); a call under
// capture, where loading a module is not allowed, uses the address that the
// last call outside capture on this device found.
static hkv_status noalloc_scratch(cudaStream_t stream, void **ptr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= NOALLOC_MAX_DEVICES)
        return HKV_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess)
        return HKV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (cap == cudaStreamCaptureStatusNone || g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return HKV_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return HKV_OK;
}

}  // namespace hkv

extern "C" hkv_status hkv_cascade_decode_noalloc(const hkv_problem *prob, const void *q, const hkv_tier *dense,
                                                 const hkv_tier *sparse, const int32_t *idx,
                                                 const int32_t *offsets, const int32_t *sel_len,
                                                 const hkv_tier *condensed, float *out, float *lse,
                                                 uint32_t *status, hkv_stream_t stream)
{
    // host validation, as for hkv_cascade_decode
    hkv_status s = check_problem(prob);
    if (s != HKV_OK)
        return s;
    if ((s = check_tier(dense, prob, true)) != HKV_OK || (s = check_tier(sparse, prob, true)) != HKV_OK ||
        (s = check_tier(condensed, prob, true)) != HKV_OK)
        return s;
    if (q == nullptr || !aligned(q, 16) || out == nullptr || (status != nullptr && !aligned(status, 4)))
        return HKV_ERR_INVALID_ARG;
    if (sparse != nullptr && sparse->cap > 0) {
        if (idx == nullptr || sel_len == nullptr)
            return HKV_ERR_INVALID_ARG;
        if (prob->layout == HKV_LAYOUT_FLAT_SUM && offsets == nullptr)
            return HKV_ERR_INVALID_ARG;
    }
    // The attention uses the front of the workspace layout: the status word,
    // the range words, the record slots of each unit and the records. It needs
    // at least the records of one CTA (two per warp and per unit); when the
    // array holds fewer than a full grid needs, fewer CTAs run.
    const WsLayout L = layout_of(prob, dense, sparse, condensed);
    const size_t rec = (size_t)part_stride(prob->D, prob->Hq / prob->Hkv) * sizeof(float);
    const int64_t units = (int64_t)prob->B * prob->Hkv;
    if (L.part + 2 * (size_t)(units + AT_NW) * rec > HKV_NOALLOC_SCRATCH_BYTES)
        return HKV_ERR_WORKSPACE;
    const int slots = (int)std::min<int64_t>(L.part_slots, (HKV_NOALLOC_SCRATCH_BYTES - L.part) / rec);
    const cudaStream_t st = (cudaStream_t)stream;
    if ((int64_t)prob->B * prob->Hkv == 0)
        return status ? (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) == cudaSuccess ? HKV_OK : HKV_ERR_CUDA)
                      : HKV_OK;
    void *scratch = nullptr;
    if ((s = noalloc_scratch(st, &scratch)) != HKV_OK)
        return s;
    char *base = static_cast<char *>(scratch);
    Params P = base_params(prob, L, base, dense, sparse, condensed);
    P.part_slots = slots;
    P.dense = tier_p(dense);
    P.sparse = tier_p(sparse);
    P.cond = tier_p(condensed);
    P.q = static_cast<const char *>(q);
    P.idx = const_cast<int32_t *>(idx);
    P.offsets = const_cast<int32_t *>(offsets);
    P.sel_len = const_cast<int32_t *>(sel_len);
    P.out = out;
    P.lse = lse;
    // the status word must start at zero; the previous call may have left it set
    if (cudaMemsetAsync(base, 0, sizeof(uint32_t), st) != cudaSuccess)
        return HKV_ERR_CUDA;
    set_row_maps(prob, sparse, P);
    if ((s = dispatch<RunAttn>(prob, P, st, false)) != HKV_OK)
        return s;
    if (status != nullptr &&
        cudaMemcpyAsync(status, base, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return HKV_ERR_CUDA;
    return HKV_OK;
}

// =============================================================================
// KV append with the dense-window roll ([TS 2.A] pipeline step 1)
//
// The newest token enters the dense window of each unit. The window is a ring
// of cap slots: while it has room the token takes slot len; once it is full
// the token replaces the oldest one, at slot head, and head advances. The
// token that leaves the window is appended to the sparse tier (so the sparse
// tier stays in age order), or dropped and reported when that tier is full.
// With no window (cap 0) the new token goes straight to the sparse tier.
// =============================================================================

namespace hkv {

struct AppendP {
    const char *k_new, *v_new;  // [units, D] rows of row_bytes
    char *dk, *dv, *sk, *sv;    // tier storage, written in place
    int64_t dsb, dsh, dst, ssb, ssh, sst;  // byte strides
    int32_t wcap, ncap;
    int32_t *dlen, *slen, *head, *dropped;
    int32_t Hkv, units, chunks;  // chunks: 16-byte pieces of one row
    uint32_t *status;
};

constexpr int APPEND_WARPS = 8;

// One warp per unit. Lane l moves the 16-byte pieces l, l+32, ... of the K row
// followed by the V row; each piece is read and rewritten by the same lane, so
// the old window row is in registers before its slot is overwritten.
__global__ void __launch_bounds__(APPEND_WARPS * 32) k_append(const __grid_constant__ AppendP A)
{
    const int u = blockIdx.x * APPEND_WARPS + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (u >= A.units)
        return;
    const int b = u / A.Hkv, h = u - b * A.Hkv;
    const int W = A.wcap > 0 ? __ldcg(A.dlen + u) : 0;
    const int n = A.ncap > 0 ? __ldcg(A.slen + u) : 0;
    const int hd = A.wcap > 0 ? __ldcg(A.head + u) : 0;
    const bool bad_len = W < 0 || W > A.wcap || n < 0 || n > A.ncap;
    const bool bad_head = A.wcap > 0 && (hd < 0 || hd >= A.wcap);
    if (bad_len || bad_head) {
        // a corrupt unit is left as it is
        if (lane == 0) {
            atomicOr(A.status, (bad_len ? HKV_DEV_LEN_CLAMPED : 0u) | (bad_head ? HKV_DEV_BAD_INDEX : 0u));
            if (A.dropped)
                A.dropped[u] = 0;
        }
        return;
    }
    const bool room = W < A.wcap;            // the window takes the token without a roll
    const bool age_out = !room;              // a token leaves the window (or bypasses it)
    const bool keep = age_out && n < A.ncap; // ... and finds room in the sparse tier
    const int dslot = room ? W : hd;
    const int64_t noff = (int64_t)u * A.chunks * 16;
    const int64_t doff = (int64_t)b * A.dsb + (int64_t)h * A.dsh + (int64_t)dslot * A.dst;
    const int64_t soff = (int64_t)b * A.ssb + (int64_t)h * A.ssh + (int64_t)n * A.sst;
    for (int c = lane; c < 2 * A.chunks; c += 32) {
        const bool isv = c >= A.chunks;
        const int off = (c - (isv ? A.chunks : 0)) * 16;
        const uint4 fresh = __ldg(reinterpret_cast<const uint4 *>((isv ? A.v_new : A.k_new) + noff + off));
        uint4 *srow = reinterpret_cast<uint4 *>((isv ? A.sv : A.sk) + soff + off);
        if (A.wcap > 0) {
            uint4 *slot = reinterpret_cast<uint4 *>((isv ? A.dv : A.dk) + doff + off);
            if (keep)
                *srow = *slot;  // the oldest row moves on
            *slot = fresh;
        } else if (keep) {
            *srow = fresh;
        }
    }
    if (lane == 0) {
        if (room)
            A.dlen[u] = W + 1;
        else if (A.wcap > 0)
            A.head[u] = hd + 1 == A.wcap ? 0 : hd + 1;
        if (keep)
            A.slen[u] = n + 1;
        if (age_out && !keep)
            atomicOr(A.status, HKV_DEV_SPARSE_FULL);
        if (A.dropped)
            A.dropped[u] = age_out && !keep;
    }
}

}  // namespace hkv

extern "C" hkv_status hkv_append(const hkv_problem *prob, const void *k_new, const void *v_new,
                                 const hkv_tier *dense, int32_t *dense_head, const hkv_tier *sparse,
                                 int32_t *dropped, void *ws, size_t ws_bytes, hkv_stream_t stream)
{
    hkv_status s = check_problem(prob);
    if (s != HKV_OK)
        return s;
    if ((s = check_tier(dense, prob, true)) != HKV_OK || (s = check_tier(sparse, prob, true)) != HKV_OK)
        return s;
    if (ws == nullptr || !aligned(ws, 256) || ws_bytes < 256)
        return HKV_ERR_WORKSPACE;
    if (k_new == nullptr || v_new == nullptr || !aligned(k_new, 16) || !aligned(v_new, 16))
        return HKV_ERR_INVALID_ARG;
    const int wcap = dense ? dense->cap : 0, ncap = sparse ? sparse->cap : 0;
    if (wcap > 0 && (dense_head == nullptr || !aligned(dense_head, 4)))
        return HKV_ERR_INVALID_ARG;
    if (dropped != nullptr && !aligned(dropped, 4))
        return HKV_ERR_INVALID_ARG;
    const int64_t units = (int64_t)prob->B * prob->Hkv;
    if (units == 0)
        return HKV_OK;
    const int es = es_of(prob->dtype);
    AppendP A{};
    A.k_new = static_cast<const char *>(k_new);
    A.v_new = static_cast<const char *>(v_new);
    if (wcap > 0) {
        A.dk = static_cast<char *>(const_cast<void *>(dense->k));
        A.dv = static_cast<char *>(const_cast<void *>(dense->v));
        A.dsb = dense->stride_b * es;
        A.dsh = dense->stride_h * es;
        A.dst = dense->stride_t * es;
        A.dlen = const_cast<int32_t *>(dense->len);
        A.head = dense_head;
    }
    if (ncap > 0) {
        A.sk = static_cast<char *>(const_cast<void *>(sparse->k));
        A.sv = static_cast<char *>(const_cast<void *>(sparse->v));
        A.ssb = sparse->stride_b * es;
        A.ssh = sparse->stride_h * es;
        A.sst = sparse->stride_t * es;
        A.slen = const_cast<int32_t *>(sparse->len);
    }
    A.wcap = wcap;
    A.ncap = ncap;
    A.dropped = dropped;
    A.Hkv = prob->Hkv;
    A.units = (int32_t)units;
    A.chunks = prob->D * es / 16;
    A.status = static_cast<uint32_t *>(ws);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((units + APPEND_WARPS - 1) / APPEND_WARPS));
    cfg.blockDim = dim3(APPEND_WARPS * 32);
    cfg.stream = (cudaStream_t)stream;
    if (cudaLaunchKernelEx(&cfg, k_append, A) != cudaSuccess)
        return HKV_ERR_CUDA;
    g_launches.fetch_add(1);
    return HKV_OK;
}

// =============================================================================
// Condensed-tier formation ([TS 2.A] Tier 3 "the oldest blocks are further
// compressed into constant-sized storage via eviction or weighted merging";
// pipeline step 4)
//
// A unit whose sparse tier holds at least max(trigger, block) tokens gives up
// its oldest `block` tokens (sparse slots 0 .. block-1; the tier is in age
// order). They become one condensed slot after the existing ones: under MERGE
// the weighted mean of the block's K and V rows, weighted by the tokens'
// calibrated probabilities a_j = exp(beta (z_j - m) - logZ) under the step's
// scores, with weight sum_j a_j; under EVICT a copy of the block's most
// important token (largest score, the older one on ties) with weight a_j. A
// full condensed tier first merges its two oldest slots (MERGE; a one-slot tier
// folds the block into its slot) or drops its oldest slot (EVICT). The sparse
// tier then moves down by `block` rows. Means are float64 sums in slot order
// (multiply, then add: no fused multiply-add), divided once and rounded once to
// the element type, nearest with ties to even.
//
// Each unit is worked by a cluster of COND_CTAS CTAs; CTA r owns bytes
// [r RB / COND_CTAS, (r+1) RB / COND_CTAS) of every K and V row (RB bytes per
// row), for the mean and for the move alike, so the CTAs never touch the same
// byte. They meet once, at a cluster barrier before the lengths and weights
// (read by all of them at the start) are updated.
// =============================================================================

namespace hkv {

constexpr int COND_CTAS = 4;
constexpr int COND_NT = 256;
constexpr int COND_STAGE = 32768;  // bytes one CTA moves per batch (its K and V slices)

struct CondP {
    char *sk, *sv, *ck, *cv;               // tier storage, written in place
    int64_t ssb, ssh, sst, csb, csh, cst;  // byte strides
    int32_t ncap, ccap;
    int32_t *slen, *clen, *done;
    float *cw;                             // [units, ccap] condensed-slot weights
    const float *z, *m, *logZ, *inv_temp;
    int64_t z_stride;
    int32_t Hkv, units, D, es, block, trigger, policy;
    uint32_t *status;
};

struct __align__(16) CondSmem {
    double a[HKV_CONDENSE_MAX_BLOCK];  // the block's weights
    unsigned char stage[COND_STAGE];   // one batch of the move
    int32_t jstar;
};

// The bf16 value nearest x, ties to an even last mantissa bit, from the double
// directly (a detour through float would round twice): integer rounding of the
// 53-bit significand to 8 bits, or to the fixed 2^-133 spacing below 2^-126.
__device__ __forceinline__ uint16_t bf16_from_double(double x)
{
    const unsigned long long bits = (unsigned long long)__double_as_longlong(x);
    const uint16_t sign = (uint16_t)((bits >> 48) & 0x8000u);
    const unsigned long long mag = bits & 0x7fffffffffffffffull;
    if (mag >= 0x7ff0000000000000ull)  // inf or NaN
        return (uint16_t)(sign | 0x7f80u | (mag > 0x7ff0000000000000ull ? 0x40u : 0u));
    const int e = (int)(mag >> 52) - 1023;
    if (e < -134)  // below a quarter of the smallest bf16 step: 0 (double subnormals included)
        return sign;
    const unsigned long long sig = (mag & 0xfffffffffffffull) | (1ull << 52);
    // drop s low bits: 45 for a normal bf16 (8 significant bits kept), more below 2^-126
    const int s = e >= -126 ? 45 : 45 + (-126 - e);
    unsigned long long keep = sig >> s;
    const unsigned long long rem = sig & ((1ull << s) - 1ull), half = 1ull << (s - 1);
    if (rem > half || (rem == half && (keep & 1ull)))
        ++keep;
    if (e < -126)  // subnormal (or the smallest normal, if rounding carried): keep is the whole pattern
        return (uint16_t)(sign | (uint16_t)keep);
    int ee = e;
    if (keep == 256ull) {
        keep = 128ull;
        ++ee;
    }
    if (ee > 127)
        return (uint16_t)(sign | 0x7f80u);
    return (uint16_t)(sign | (uint16_t)((ee + 127) << 7) | (uint16_t)(keep & 0x7fu));
}

__device__ __forceinline__ double cond_load(const char *row, int e, int es)
{
    if (es == 2)
        return (double)__uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t *>(row + 2 * e)) << 16);
    return (double)*reinterpret_cast<const float *>(row + 4 * e);
}

__device__ __forceinline__ void cond_store(char *row, int e, int es, double v)
{
    if (es == 2)
        *reinterpret_cast<uint16_t *>(row + 2 * e) = bf16_from_double(v);
    else
        *reinterpret_cast<float *>(row + 4 * e) = __double2float_rn(v);
}

__device__ __forceinline__ void cond_copy_elem(char *dst, const char *src, int e, int es)
{
    if (es == 2)
        *reinterpret_cast<uint16_t *>(dst + 2 * e) = *reinterpret_cast<const uint16_t *>(src + 2 * e);
    else
        *reinterpret_cast<uint32_t *>(dst + 4 * e) = *reinterpret_cast<const uint32_t *>(src + 4 * e);
}

__global__ void __cluster_dims__(COND_CTAS, 1, 1) __launch_bounds__(COND_NT)
    k_condense(const __grid_constant__ CondP P)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    CondSmem &sm = *reinterpret_cast<CondSmem *>(smem_raw);
    auto cluster = cooperative_groups::this_cluster();
    const int r = (int)cluster.block_rank();
    const int u = blockIdx.x / COND_CTAS;
    const int b = u / P.Hkv, h = u - b * P.Hkv;
    const int n = __ldcg(P.slen + u);
    const int C0 = P.ccap > 0 ? __ldcg(P.clen + u) : 0;
    if (n < 0 || n > P.ncap || C0 < 0 || C0 > P.ccap) {  // a corrupt unit is left as it is
        if (r == 0 && threadIdx.x == 0) {
            atomicOr(P.status, HKV_DEV_LEN_CLAMPED);
            if (P.done)
                P.done[u] = 0;
        }
        return;
    }
    const int blk = P.block;
    if (n < max(max(P.trigger, blk), 1)) {
        if (r == 0 && threadIdx.x == 0 && P.done)
            P.done[u] = 0;
        return;
    }
    char *sk = P.sk + (int64_t)b * P.ssb + (int64_t)h * P.ssh;
    char *sv = P.sv + (int64_t)b * P.ssb + (int64_t)h * P.ssh;
    char *ck = P.ccap > 0 ? P.ck + (int64_t)b * P.csb + (int64_t)h * P.csh : nullptr;
    char *cv = P.ccap > 0 ? P.cv + (int64_t)b * P.csb + (int64_t)h * P.csh : nullptr;
    float *cw = P.ccap > 0 ? P.cw + (int64_t)u * P.ccap : nullptr;

    // the block's weights (and, for EVICT, its first highest-scoring token)
    double beta = 1.0;
    if (P.inv_temp != nullptr) {
        const float bt = __ldcg(P.inv_temp + u);
        if (!(bt >= 0.0f) || isinf(bt)) {
            if (r == 0 && threadIdx.x == 0)
                atomicOr(P.status, HKV_DEV_BAD_TEMP);
        } else {
            beta = (double)bt;
        }
    }
    const float *zu = P.z != nullptr ? P.z + (int64_t)u * P.z_stride : nullptr;
    const double mu = zu ? (double)__ldcg(P.m + u) : 0.0, lz = zu ? (double)__ldcg(P.logZ + u) : 0.0;
    for (int j = threadIdx.x; j < blk; j += COND_NT)
        sm.a[j] = zu ? exp(__dsub_rn(__dmul_rn(beta, __dsub_rn((double)__ldcg(zu + j), mu)), lz)) : 1.0;
    if (threadIdx.x == 0)
        sm.jstar = 0;
    __syncthreads();
    if (P.policy == HKV_CONDENSE_EVICT && zu != nullptr) {
        // first maximum: the largest (score, -index) pair
        unsigned long long best = 0ull;
        for (int j = threadIdx.x; j < blk; j += COND_NT) {
            const unsigned long long key = ((unsigned long long)(~score_key(__ldcg(zu + j))) << 32) |
                                           (uint32_t)(0x7fffffff - j);
            best = key > best ? key : best;
        }
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long y = __shfl_xor_sync(0xffffffffu, best, o);
            best = y > best ? y : best;
        }
        __shared__ unsigned long long wbest[COND_NT / 32];
        if ((threadIdx.x & 31) == 0)
            wbest[threadIdx.x >> 5] = best;
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned long long m_ = 0ull;
            for (int w = 0; w < COND_NT / 32; ++w)
                m_ = wbest[w] > m_ ? wbest[w] : m_;
            sm.jstar = 0x7fffffff - (int)(uint32_t)m_;
        }
        __syncthreads();
    }

    // this CTA's elements of a row: NE of K, then NE of V
    const int NE = P.D / COND_CTAS;
    const int e0 = r * NE;
    int C = C0;             // slot of the new condensed entry
    bool fold = false;      // one-slot MERGE tier: the old slot joins the block's mean
    if (P.ccap > 0) {
        const bool full = C0 >= P.ccap;
        if (P.policy == HKV_CONDENSE_MERGE && full && P.ccap >= 2) {
            const double w0 = (double)cw[0], w1 = (double)cw[1];
            const bool eq = !(__dadd_rn(__dadd_rn(0.0, w0), w1) > 0.0);
            const double a0 = eq ? 1.0 : w0, a1 = eq ? 1.0 : w1;
            for (int t = threadIdx.x; t < 2 * NE; t += COND_NT) {
                char *base = t < NE ? ck : cv;
                const int e = e0 + (t < NE ? t : t - NE);
                const double x0 = cond_load(base, e, P.es), x1 = cond_load(base + P.cst, e, P.es);
                double num = __dadd_rn(0.0, __dmul_rn(a0, x0));  // sums start at +0, as in any plain loop
                num = __dadd_rn(num, __dmul_rn(a1, x1));
                const double den = __dadd_rn(__dadd_rn(0.0, a0), a1);
                cond_store(base, e, P.es, __ddiv_rn(num, den));
                for (int i = 1; i + 1 < P.ccap; ++i)  // the later slots move down by one
                    cond_copy_elem(base + (int64_t)i * P.cst, base + (int64_t)(i + 1) * P.cst, e, P.es);
            }
            C = P.ccap - 1;
        } else if (P.policy == HKV_CONDENSE_MERGE && full) {
            fold = true;
            C = 0;
        } else if (full) {  // EVICT: the oldest slot goes
            for (int t = threadIdx.x; t < 2 * NE; t += COND_NT) {
                char *base = t < NE ? ck : cv;
                const int e = e0 + (t < NE ? t : t - NE);
                for (int i = 0; i + 1 < P.ccap; ++i)
                    cond_copy_elem(base + (int64_t)i * P.cst, base + (int64_t)(i + 1) * P.cst, e, P.es);
            }
            C = P.ccap - 1;
        }
        if (P.policy == HKV_CONDENSE_MERGE) {
            // weights in slot order: the folded slot's first, then the block's
            const double wf = fold ? (double)cw[0] : 0.0;
            double S = fold ? __dadd_rn(0.0, wf) : 0.0;
            for (int j = 0; j < blk; ++j)
                S = __dadd_rn(S, sm.a[j]);
            const bool eq = !(S > 0.0);
            for (int t = threadIdx.x; t < 2 * NE; t += COND_NT) {
                const bool isk = t < NE;
                const char *src = isk ? sk : sv;
                char *dst = (isk ? ck : cv) + (int64_t)C * P.cst;
                const int e = e0 + (isk ? t : t - NE);
                double num = 0.0, den = 0.0;
                if (fold) {
                    const double a_ = eq ? 1.0 : wf;
                    num = __dadd_rn(num, __dmul_rn(a_, cond_load(dst, e, P.es)));
                    den = __dadd_rn(den, a_);
                }
#pragma unroll 4
                for (int j = 0; j < blk; ++j) {
                    const double a_ = eq ? 1.0 : sm.a[j];
                    num = __dadd_rn(num, __dmul_rn(a_, cond_load(src + (int64_t)j * P.sst, e, P.es)));
                    den = __dadd_rn(den, a_);
                }
                cond_store(dst, e, P.es, __ddiv_rn(num, den));
            }
        } else {
            const int js = sm.jstar;
            for (int t = threadIdx.x; t < 2 * NE; t += COND_NT) {
                const bool isk = t < NE;
                const int e = e0 + (isk ? t : t - NE);
                cond_copy_elem((isk ? ck : cv) + (int64_t)C * P.cst, (isk ? sk : sv) + (int64_t)js * P.sst, e, P.es);
            }
        }
    }
    __syncthreads();  // the block's rows are read; the move may overwrite them

    // the sparse tier moves down by blk rows: batches staged in shared memory
    // (a batch's rows are all read before any is written, and a later batch
    // reads only rows above everything written so far)
    const int QB = NE * P.es;          // this CTA's bytes of one row of K (and of V)
    const int QC = QB / 16;            // ... in 16-byte chunks
    const int rows_per_batch = COND_STAGE / (2 * QB);
    const int left = n - blk;
    for (int r0 = 0; r0 < left; r0 += rows_per_batch) {
        const int rows = min(rows_per_batch, left - r0);
        const int chunks = rows * 2 * QC;
        for (int c = threadIdx.x; c < chunks; c += COND_NT) {
            const int row = c / (2 * QC), q = c - row * 2 * QC;
            const bool isk = q < QC;
            const char *src = (isk ? sk : sv) + (int64_t)(r0 + blk + row) * P.sst + e0 * P.es + (isk ? q : q - QC) * 16;
            *reinterpret_cast<uint4 *>(sm.stage + c * 16) = __ldcs(reinterpret_cast<const uint4 *>(src));
        }
        __syncthreads();
        for (int c = threadIdx.x; c < chunks; c += COND_NT) {
            const int row = c / (2 * QC), q = c - row * 2 * QC;
            const bool isk = q < QC;
            char *dst = (isk ? sk : sv) + (int64_t)(r0 + row) * P.sst + e0 * P.es + (isk ? q : q - QC) * 16;
            *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(sm.stage + c * 16);
        }
        __syncthreads();
    }
    // every CTA of the unit has read the lengths and weights: update them
    cluster.sync();
    if (r == 0 && threadIdx.x == 0) {
        P.slen[u] = n - blk;
        if (P.ccap > 0) {
            if (P.policy == HKV_CONDENSE_MERGE) {
                if (C0 >= P.ccap && P.ccap >= 2) {
                    cw[0] = __double2float_rn(__dadd_rn(__dadd_rn(0.0, (double)cw[0]), (double)cw[1]));
                    for (int i = 1; i + 1 < P.ccap; ++i)
                        cw[i] = cw[i + 1];
                }
                double S = fold ? __dadd_rn(0.0, (double)cw[0]) : 0.0;
                for (int j = 0; j < blk; ++j)
                    S = __dadd_rn(S, sm.a[j]);
                cw[C] = __double2float_rn(S);
            } else {
                if (C0 >= P.ccap)
                    for (int i = 0; i + 1 < P.ccap; ++i)
                        cw[i] = cw[i + 1];
                cw[C] = __double2float_rn(sm.a[sm.jstar]);
            }
            P.clen[u] = C + 1;
        }
        if (P.done)
            P.done[u] = 1;
    }
}

}  // namespace hkv

extern "C" hkv_status hkv_condense(const hkv_problem *prob, const hkv_tier *sparse, const hkv_tier *condensed,
                                   float *cond_w, const float *z, int64_t z_stride, const float *m,
                                   const float *logZ, int32_t block, int32_t trigger,
                                   hkv_condense_policy policy, int32_t *done, void *ws, size_t ws_bytes,
                                   hkv_stream_t stream)
{
    hkv_status s = check_problem(prob);
    if (s != HKV_OK)
        return s;
    if (sparse == nullptr)
        return HKV_ERR_INVALID_ARG;
    if ((s = check_tier(sparse, prob, true)) != HKV_OK || (s = check_tier(condensed, prob, true)) != HKV_OK)
        return s;
    if (ws == nullptr || !aligned(ws, 256) || ws_bytes < 256)
        return HKV_ERR_WORKSPACE;
    const int ncap = sparse->cap, ccap = condensed ? condensed->cap : 0;
    if (block < 1 || block > HKV_CONDENSE_MAX_BLOCK || block > ncap || trigger < 0 ||
        (policy != HKV_CONDENSE_MERGE && policy != HKV_CONDENSE_EVICT))
        return HKV_ERR_INVALID_ARG;
    if (ccap > 0 && (cond_w == nullptr || !aligned(cond_w, 4)))
        return HKV_ERR_INVALID_ARG;
    const bool scores = z != nullptr || m != nullptr || logZ != nullptr;
    if (scores && (z == nullptr || m == nullptr || logZ == nullptr || !aligned(z, 4) || z_stride < ncap))
        return HKV_ERR_INVALID_ARG;
    if (done != nullptr && !aligned(done, 4))
        return HKV_ERR_INVALID_ARG;
    const int64_t units = (int64_t)prob->B * prob->Hkv;
    if (units == 0 || ncap == 0)
        return HKV_OK;
    const int es = es_of(prob->dtype);
    CondP P{};
    P.sk = static_cast<char *>(const_cast<void *>(sparse->k));
    P.sv = static_cast<char *>(const_cast<void *>(sparse->v));
    P.ssb = sparse->stride_b * es;
    P.ssh = sparse->stride_h * es;
    P.sst = sparse->stride_t * es;
    P.slen = const_cast<int32_t *>(sparse->len);
    if (ccap > 0) {
        P.ck = static_cast<char *>(const_cast<void *>(condensed->k));
        P.cv = static_cast<char *>(const_cast<void *>(condensed->v));
        P.csb = condensed->stride_b * es;
        P.csh = condensed->stride_h * es;
        P.cst = condensed->stride_t * es;
        P.clen = const_cast<int32_t *>(condensed->len);
    }
    P.ncap = ncap;
    P.ccap = ccap;
    P.cw = cond_w;
    P.z = scores ? z : nullptr;
    P.m = scores ? m : nullptr;
    P.logZ = scores ? logZ : nullptr;
    P.z_stride = z_stride;
    P.inv_temp = prob->inv_temp;
    P.done = done;
    P.Hkv = prob->Hkv;
    P.units = (int32_t)units;
    P.D = prob->D;
    P.es = es;
    P.block = block;
    P.trigger = trigger;
    P.policy = (int32_t)policy;
    P.status = static_cast<uint32_t *>(ws);
    const size_t smem = sizeof(CondSmem);
    if ((s = prepare((const void *)k_condense, COND_NT, smem, nullptr)) != HKV_OK)
        return s;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(units * COND_CTAS));
    cfg.blockDim = dim3(COND_NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = (cudaStream_t)stream;
    if (cudaLaunchKernelEx(&cfg, k_condense, P) != cudaSuccess)
        return HKV_ERR_CUDA;
    g_launches.fetch_add(1);
    return HKV_OK;
}
