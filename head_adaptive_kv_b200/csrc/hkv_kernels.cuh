// hkv_kernels.cuh -- device code of the HARD-KV Cascade Cache decode step.
//
// Sources: [Abstract] = arXiv abstract on the mlsanity.com page "HARD-KV:
// Head-Adaptive Regularization for Decoding-time KV Compression"; [TS 2.A],
// [TS 2.B], [TS 2.C] = sections "Cascade Cache Hierarchy", "Logits Calibration
// Mechanism", "System-Aware Index Regularization" of the gist.science Technical
// Summary of that paper.
//
// Two kinds of kernels:
//  - streaming kernels (scoring, attention): every warp runs its own copy
//    pipeline over a contiguous share of the kernel's work (a static, balanced
//    partition: no tickets, no producer warp). It keeps several stages in
//    flight in its own ring of shared-memory slots, armed and filled by the
//    warp itself with 1-D TMA bulk copies (one per contiguous run, or one per
//    gathered row), completion on one mbarrier per slot.
//  - per-unit kernels (selection, compaction, calibration, layout): one CTA of
//    SEL_THREADS threads per (sequence, KV head).
// No tensor cores: a one-query decode is a GEMV (about 4 flop per byte), bound
// by HBM bandwidth.
#pragma once

#include <cfloat>
#include <cooperative_groups.h>

#include "hkv_device.cuh"

namespace hkv {


constexpr int SC_SLOT = 8192;             // scoring: bytes per stage (K rows)
// scoring: warps per CTA and ring slots per warp (192 KB of slots per CTA);
// eight query heads per group keep twice the query registers per lane, so
// they run fewer warps with more slots each
__host__ __device__ constexpr int sc_nw(int G) { return G >= 8 ? 8 : 12; }
__host__ __device__ constexpr int sc_stages(int G) { return G >= 8 ? 3 : 2; }
constexpr int AT_NW = 8;                  // attention: warps per CTA
constexpr int AT_SLOT = 8192;             // attention: bytes per stage (K rows, then as many V rows)
constexpr int AT_STAGES = 3;              // attention: ring slots per warp
constexpr int SC_FLOATS = 256;            // per-warp logits of one attention stage
constexpr bool ATTN_UNROLL_QK = true;     // attention: unroll the logit batches of a full stage
constexpr int PREFIX_CAP = 1024;          // attention: units whose token prefixes fit in shared memory
constexpr int SEL_THREADS = 512;          // per-unit kernels
constexpr float LOG2E = 1.4426950408889634f;

struct TierP {
    const char *k, *v;
    int64_t sb, sh, st;  // element strides
    int32_t cap;
    const int32_t *len;  // nullptr = empty tier
};

struct Params {
    int32_t B, Hq, Hkv, D, G, units;
    float scale, p;
    int32_t bmin, bmax, layout;
    const float *inv_temp, *p_unit;
    const char *q;
    TierP dense, sparse, cond;
    // outputs
    float *z;
    int64_t z_stride;
    int32_t *sel_len;
    hkv_cut *cut;
    int32_t *idx;        // PAD_MAX rows (caller's idx or workspace rows) / caller's FLAT_SUM idx
    int32_t *idx_user;   // the caller's idx in its own layout (flatten kernel)
    int32_t *offsets;
    float *out, *lse, *m_out, *logZ_out, *P_out;
    char *k_out, *v_out;
    // per-head logits scale * q_g . k_j of every sparse token, written by the
    // scorer and read back by the attention for the selected tokens (hkv_step
    // only, else nullptr): token j of unit u at logit + (u cap + j) * LG
    float *logit;
    // workspace
    uint32_t *ctl;        // [0] status word
    uint32_t *urange;     // [units][2] score range of each unit as order keys (step only, else nullptr)
    int32_t *rec_range;   // [units][4] first and last record slot of each unit on attention lines A and B
    float *part;          // [part_slots * part_stride] attention records
    int32_t part_slots;   // record slots: 2 x (streaming warps of the attention grid + units)
    int32_t attn_prefix;  // attention partition over actual tokens (units <= PREFIX_CAP, lines < 2^31), else over capacity
    int32_t attn_a_ctas;  // attention CTAs that share line A (the first ones, which start while the selection runs)
    int32_t unit_ctas;    // CTAs of the selection kernel before the attention (units, or more when split)
    int32_t have_range;   // per-unit kernel: urange holds the units' score ranges
    int32_t do_select, do_compact;  // per-unit kernel: which steps to run
    int32_t withhold;     // fault injection: streaming warps never arm their stages
    // fitted temperature: per-unit entropy target in (nullptr: from the logit
    // records), target out, fitted inverse temperature out
    const float *h_target;
    float *h_out, *beta_out;
    uint64_t wait_ns;
    // Rewrite Cache vs Sparse Loading (hkv_step_mti; nullptr elsewhere): steps
    // each unit's rewrite still serves (> 0: the unit reuses it this step),
    // the rewrite buffer (rows in its len) and the token indices of its rows
    const int32_t *mti_left;
    TierP rw;
    const int32_t *rw_idx;
    // kernel timeline (hkv_set_timeline; nullptr when off): per kernel kind,
    // the complement of its earliest start and its latest end (global timer)
    unsigned long long *tl;
    // a plainly laid out sparse tier: its V rows (vmap_ok; hkv_step and the
    // attention calls) and K rows (kmap_ok; the attention calls, which gather
    // both) as 2-D tensor maps (row u cap + j = token j of unit u, D elements,
    // box one row high), for the attention's four-row TMA gathers of selected
    // rows
    int32_t vmap_ok, kmap_ok;
    CUtensorMap vmap, kmap;
};

// Kernel kinds of the timeline (index of their start word; the end word is 8 on).
enum : int { TL_SCORE = 0, TL_UNIT = 1, TL_ATTN = 2, TL_MERGE = 3, TL_FLAT = 4, TL_FIT = 5, TL_MTI = 6 };

// A CTA's start and end on the timeline: starts are kept as complements under
// atomicMax, so that zeroed words mean "nothing recorded" for both.
__device__ __forceinline__ void tl_start(unsigned long long *tl, int kind)
{
    if (tl != nullptr && threadIdx.x == 0)
        atomicMax(tl + kind, ~(unsigned long long)global_ns());
}

__device__ __forceinline__ void tl_end(unsigned long long *tl, int kind)
{
    if (tl != nullptr) {
        __syncthreads();
        if (threadIdx.x == 0)
            atomicMax(tl + 8 + kind, (unsigned long long)global_ns());
    }
}

__device__ __forceinline__ Ctl make_ctl(const Params &P) { return Ctl{P.ctl, P.wait_ns}; }

__device__ __forceinline__ int tier_len(const TierP &t, int u, const Ctl &c)
{
    if (t.len == nullptr)
        return 0;
    int n = __ldcg(t.len + u);
    if (n < 0 || n > t.cap) {
        raise_flag(c, HKV_DEV_LEN_CLAMPED);
        n = n < 0 ? 0 : t.cap;
    }
    return n;
}

__device__ __forceinline__ float unit_beta(const Params &P, int u, const Ctl &c)
{
    if (P.inv_temp == nullptr)
        return 1.0f;
    const float b = __ldcg(P.inv_temp + u);
    if (!(b >= 0.0f) || isinf(b)) {
        raise_flag(c, HKV_DEV_BAD_TEMP);
        return 1.0f;
    }
    return b;
}

__device__ __forceinline__ float unit_p(const Params &P, int u, const Ctl &c)
{
    if (P.p_unit == nullptr)
        return P.p;
    const float p = __ldcg(P.p_unit + u);
    if (p != p) {
        raise_flag(c, HKV_DEV_BAD_P);
        return 1.0f;
    }
    return p;
}

// The budget of a unit as the attention sees it (clamped into [0, min(n, bmax)]).
__device__ __forceinline__ int unit_budget(const Params &P, int u, int n, const Ctl &c)
{
    if (P.sparse.len == nullptr)
        return 0;
    int k = __ldcg(P.sel_len + u);
    if (k < 0 || k > n || k > P.bmax) {
        raise_flag(c, HKV_DEV_BAD_INDEX);
        k = max(0, min(k, min(n, P.bmax)));
    }
    return k;
}

// Floats of one attention record (o[G][D], m[G], l[G]), padded to a multiple of 4.
__host__ __device__ constexpr int part_stride(int D, int G) { return (G * (D + 2) + 3) / 4 * 4; }

// Floats of one token's logit record (G logits, padded to 16 bytes).
__host__ __device__ constexpr int logit_floats(int G) { return (G + 3) / 4 * 4; }

// Order-preserving 32-bit keys of floats (larger float, larger key), so that
// atomicMax on keys takes the maximum of floats. Key 0 means "none".
__device__ __forceinline__ uint32_t ord_key(float x)
{
    const uint32_t b = __float_as_uint(x);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ord_val(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Compile-time geometry of a (element size, head dim, group size) instance.
// A K row is read by LPR lanes, each taking CPL 16-byte chunks (chunk l % LPR
// and chunk l % LPR + LPR), so each 8-lane phase of a 16-byte shared load
// covers 128 contiguous bytes (no bank conflicts).
template <int ES, int D, int G>
struct Geo {
    static constexpr int ROWB = D * ES;                   // bytes of one K or V row
    static constexpr int CPL = ROWB >= 256 ? 2 : 1;       // 16-byte chunks per lane per row
    static constexpr int LPR = ROWB / (16 * CPL);         // lanes per row
    static constexpr int RPW = 32 / LPR;                  // rows per warp iteration
    static constexpr int VEC = 16 / ES;                   // elements per 16-byte chunk
    static constexpr int NP = CPL * VEC / 2;              // float2 pairs per lane per row
    static constexpr int ITB = 32 * 16 * CPL;             // bytes of one warp iteration
    static constexpr int SITERS = SC_SLOT / ITB;          // iterations per scoring stage
    static constexpr int AITERS = (AT_SLOT / 2) / ITB;    // iterations over an attention stage's keys
    static constexpr int NB0 = LPR / G;
    static constexpr int NB0S = NB0 < SITERS ? NB0 : SITERS;
    static constexpr int NB = NB0S < AITERS ? NB0S : AITERS;  // iterations reduced together
    static constexpr int NV = NB * G;                     // partial sums per lane before reduction
    static constexpr int REP = LPR / NV;                  // lanes holding the same sum afterwards
    static constexpr int SROWS = SC_SLOT / ROWB;          // rows per scoring stage
    static constexpr int ATOK = (AT_SLOT / 2) / ROWB;     // tokens per attention stage (K and V rows)
    // a stage of selected tokens read with the scorer's logits holds no K rows:
    // room for 32 logit records, then BTOK V rows from byte VOFF_B (fewer,
    // fuller stages: a warp's share of the selection is only a few stages long)
    static constexpr int VOFF_B = 32 * logit_floats(G) * 4;
    static constexpr int BTOK0 = (AT_SLOT - VOFF_B) / ROWB;
    static constexpr int BTOK = (BTOK0 < 32 ? BTOK0 : 32) / 4 * 4;  // whole groups of four rows
    static constexpr int DPL = D / 32;                    // PV: head-dim elements per lane
    static_assert(G >= 1 && G <= LPR, "group size must not exceed lanes per row");
    static_assert(ATOK * G <= SC_FLOATS && ATOK <= 32, "stage sizes");
    static_assert(ATOK * logit_floats(G) * 4 <= AT_SLOT / 2, "logit records of a stage");
    static_assert(BTOK * G <= SC_FLOATS && BTOK >= ATOK && VOFF_B % 16 == 0, "stages of selected tokens");
    static_assert(ATOK % 4 == 0, "K and V stages in whole groups of four rows");
    static_assert(SITERS % NB == 0 && AITERS % NB == 0 && LPR % NV == 0, "iteration batches");
};

// =============================================================================
// Streaming engine
// =============================================================================

enum : int32_t { SD_FIRST = 1, SD_LAST = 2, SD_GATHER = 4, SD_ARMED = 8, SD_LOGIT = 16, SD_LINEB = 32 };

// Trace builds (-DHKV_TRACE): per warp trace slot base s (4 slots), the issue
// and landing times of its first 12 stages at TRACE_STAGES + 8 s + 2 i (+1).
[[maybe_unused]] constexpr int TRACE_STAGES = 40000;

struct StageDesc {
    int32_t unit, start, count, flags;  // rows (scoring) or unit-local tokens (attention) [start, start + count)
};

template <int NW, int SLOT, int NS>
struct __align__(128) Ring {
    static constexpr int kNW = NW, kNS = NS;
    unsigned char slot[NW][NS][SLOT];
    uint64_t full[NW][NS];
    StageDesc desc[NW][NS];
};

template <class R>
__device__ __forceinline__ void ring_init(R &r)
{
    if (threadIdx.x == 0) {
        for (int w = 0; w < R::kNW; ++w)
            for (int j = 0; j < R::kNS; ++j)
                mbar_init(&r.full[w][j], 1);
        mbar_fence_init();
    }
    __syncthreads();
}

// The warp's pipeline. Job supplies (all lanes call each, warp-uniformly):
//   bool next(StageDesc &d)                  -- the warp's next stage, or false
//   void issue(const StageDesc &d, int j)    -- record d in slot j, arm it and start its copies
//   void consume(const StageDesc &d, const unsigned char *slot)
// Up to NS stages are in flight. If a wait runs out (status word set), the
// warp stops consuming, waits (bounded) for the copies it started, and returns.
template <class Job, class R>
__device__ uint32_t warp_pipeline(Job &job, R &ring, const Ctl &c, int tslot = -1, uint32_t start = 0)
{
    // start: stages the warp already pushed through its ring (slot i % NS,
    // phase parity (i / NS) & 1 for the i-th stage overall)
    constexpr int NS = Job::NS;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t issued = start, consumed = start;
    StageDesc d;
    if (start > 0 && lane == 0)
        fence_proxy_async_smem();  // the warp's reads of its slots before the copies that refill them
    while (issued < start + (uint32_t)NS && job.next(d)) {
        if (issued - start < 12)
            HKV_TRACE_WARP(tslot < 0 ? -1 : TRACE_STAGES + tslot * 8 + 2 * (int)(issued - start));
        job.issue(d, (int)(issued % NS));
        ++issued;
    }
    bool ok = true;
    while (consumed < issued) {
        const int j = (int)(consumed % NS);
        if (!mbar_wait(&ring.full[w][j], (consumed / NS) & 1u, c)) {
            ok = false;
            break;
        }
        if (consumed == start)
            HKV_TRACE_WARP(tslot < 0 ? -1 : tslot + 1);
        if (consumed - start < 12)
            HKV_TRACE_WARP(tslot < 0 ? -1 : TRACE_STAGES + tslot * 8 + 2 * (int)(consumed - start) + 1);
        const StageDesc cd = ring.desc[w][j];
        job.consume(cd, ring.slot[w][j]);
        __syncwarp();
        ++consumed;
        if (job.next(d)) {
            if (lane == 0)
                fence_proxy_async_smem();  // this warp's reads of the slot before the copies that refill it
            if (issued - start < 12)
                HKV_TRACE_WARP(tslot < 0 ? -1 : TRACE_STAGES + tslot * 8 + 2 * (int)(issued - start));
            job.issue(d, j);
            ++issued;
        }
    }
    if (!ok) {
        // the copies already started must land before the CTA may exit
        for (uint32_t i = consumed; i < issued; ++i) {
            const int j = (int)(i % NS);
            if (ring.desc[w][j].flags & SD_ARMED)
                mbar_wait_bounded(&ring.full[w][j], (i / NS) & 1u, c.wait_ns);
        }
    }
    __syncwarp();
    HKV_TRACE_WARP(tslot < 0 ? -1 : tslot + 2);
    return issued;
}

// ---- warp butterfly over the LPR lanes of a row: NV partial sums per lane ->
// one full sum per lane. Reduce-scatter over the top log2(NV) lane bits, then a
// plain all-reduce over the low log2(REP) bits. Afterwards lane l holds the
// sum of value index (l % LPR) / REP.
template <int NV, int REP, int CNT>
__device__ __forceinline__ void butterfly(float (&v)[NV], int lane)
{
    if constexpr (CNT > 1) {
        constexpr int H = CNT / 2;
        constexpr int O = H * REP;  // lane bit exchanged at this level
        const bool upper = (lane & O) != 0;
#pragma unroll
        for (int i = 0; i < H; ++i) {
            const float send = upper ? v[i] : v[i + H];
            const float keep = upper ? v[i + H] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
        }
        butterfly<NV, REP, H>(v, lane);
    } else {
#pragma unroll
        for (int o = REP / 2; o >= 1; o >>= 1)
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
}

template <int ES>
__device__ __forceinline__ void unpack16(const uint4 &w, float2 *kv)
{
    if constexpr (ES == 2) {
        kv[0] = bf16x2_to_float2(w.x);
        kv[1] = bf16x2_to_float2(w.y);
        kv[2] = bf16x2_to_float2(w.z);
        kv[3] = bf16x2_to_float2(w.w);
    } else {
        kv[0] = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
        kv[1] = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
    }
}

// The lane's slice of the group's G queries of unit u (chunks l % LPR and
// l % LPR + LPR of each row), read from global memory (small, L2-resident).
template <int ES, int D, int G>
__device__ __forceinline__ void load_q(const Params &P, int u, int lane, float2 (&qv)[G][Geo<ES, D, G>::NP])
{
    using Gm = Geo<ES, D, G>;
    const int b = u / P.Hkv, h = u % P.Hkv;
    const char *qb = P.q + (int64_t)(b * P.Hq + h * G) * D * ES;
    const int c0 = lane % Gm::LPR;
    uint4 w[G][Gm::CPL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int cc = 0; cc < Gm::CPL; ++cc)
            w[g][cc] = __ldg(reinterpret_cast<const uint4 *>(qb + g * Gm::ROWB + (c0 + cc * Gm::LPR) * 16));
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int cc = 0; cc < Gm::CPL; ++cc)
            unpack16<ES>(w[g][cc], &qv[g][cc * (Gm::VEC / 2)]);
}

// One batch of NB warp iterations over staged rows: per-lane partial dot
// products with the group's queries, reduced across the LPR lanes of a row.
// Returns the lane's reduced value: row (it0 + vi / G) * RPW + lane / LPR,
// query head vi % G, with vi = (lane % LPR) / REP.
template <int ES, int D, int G>
__device__ __forceinline__ float qk_batch(const unsigned char *stage, int it0, int lane,
                                          const float2 (&qv)[G][Geo<ES, D, G>::NP])
{
    using Gm = Geo<ES, D, G>;
    const int r_in = lane / Gm::LPR, c0 = lane % Gm::LPR;
    float v[Gm::NV];
#pragma unroll
    for (int i = 0; i < Gm::NB; ++i) {
        const unsigned char *row = stage + ((it0 + i) * Gm::RPW + r_in) * Gm::ROWB;
        float2 kv[Gm::NP];
#pragma unroll
        for (int cc = 0; cc < Gm::CPL; ++cc)
            unpack16<ES>(*reinterpret_cast<const uint4 *>(row + (c0 + cc * Gm::LPR) * 16), &kv[cc * (Gm::VEC / 2)]);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int p = 0; p < Gm::NP; ++p)
                acc = ffma2(qv[g][p], kv[p], acc);
            v[i * G + g] = acc.x + acc.y;
        }
    }
    butterfly<Gm::NV, Gm::REP, Gm::NV>(v, lane);
    return v[0];
}

// Warp g of NW warps over a line of T positions takes [T g / NW, T (g+1) / NW).
__device__ __forceinline__ int64_t share_begin(int64_t g, int64_t NW, int64_t T) { return g * T / NW; }

// The warp whose share holds position t (0 <= t < T): the last g with
// share_begin(g) <= t, which is never an empty share.
__device__ __forceinline__ int64_t share_owner(int64_t t, int64_t NW, int64_t T)
{
    return ((t + 1) * NW + T - 1) / T - 1;
}

// ---- scoring ([TS 2.B] max-pooled attention logits; [TS 2.A] Tier 2) --------
//
// Work line: the rows each unit has to score, unit-major, cut into equal
// static shares, one per warp. With at most PREFIX_CAP units the line holds
// exactly those rows (a unit's length, or none for a unit that reuses a
// rewrite this step): every CTA sums the units' counts in shared memory. With
// more units the line is the capacity rows of all units, and rows past a
// unit's length are skipped. In hkv_step each warp also folds the range of
// the scores it wrote into its units' range words (atomic max of order keys),
// which the selection starts from.

// Rows unit u scores this step: its sparse length, or 0 when it reuses a rewrite.
__device__ __forceinline__ int score_len(const Params &P, int u, const Ctl &c)
{
    if (P.mti_left != nullptr && __ldcg(P.mti_left + u) > 0)
        return 0;
    return tier_len(P.sparse, u, c);
}

struct ScoreLineSmem {
    int64_t pre[PREFIX_CAP + 1];  // line position of each unit's first row
};

// Prefix layout: the units' line positions in shared memory. Returns the rows on the line.
template <int NTH>
__device__ int64_t score_prologue(const Params &P, const Ctl &c, ScoreLineSmem &L, unsigned long long *red)
{
    constexpr int UPT = (PREFIX_CAP + NTH - 1) / NTH;
    unsigned long long carry = 0;
#pragma unroll
    for (int i = 0; i < UPT; ++i) {
        if (i * NTH >= P.units)
            break;  // uniform over the CTA
        const int u = i * NTH + threadIdx.x;
        const int n = u < P.units ? score_len(P, u, c) : 0;
        unsigned long long tot;
        const unsigned long long ex = block_exclusive_scan<NTH>((unsigned long long)n, red, &tot);
        if (u < P.units)
            L.pre[u] = (int64_t)(carry + ex);
        carry += tot;
    }
    if (threadIdx.x == 0)
        L.pre[P.units] = (int64_t)carry;
    __syncthreads();
    return (int64_t)carry;
}

template <int ES, int D, int G>
struct ScoreJob {
    using Gm = Geo<ES, D, G>;
    static constexpr int NS = sc_stages(G), NW = sc_nw(G);
    using RingT = Ring<NW, SC_SLOT, NS>;
    struct Smem {
        RingT ring;
        ScoreLineSmem line;
        unsigned long long red[NW];
    };

    const Params &P;
    const Ctl &c;
    RingT &ring;
    const ScoreLineSmem *L;  // prefix layout (nullptr: capacity layout)
    uint64_t policy;
    int w, lane;
    // generator: the share's next row is row j of unit u; `left` rows remain
    int u, j;
    int64_t left;
    int gu = -1, gn = 0, last_unit = -1;
    const char *kbase = nullptr;  // K rows of unit gu (the unit of the stage last returned)
    // consumer
    float2 qv[G][Gm::NP];
    float tmax = -INFINITY, tmin = INFINITY;

    // Rows unit x holds on the line.
    __device__ __forceinline__ int span(int x) const
    {
        return L ? (int)(L->pre[x + 1] - L->pre[x]) : P.sparse.cap;
    }

    __device__ ScoreJob(const Params &P_, const Ctl &c_, RingT &ring_, const ScoreLineSmem *L_, int64_t T,
                        int64_t g, int64_t nw)
        : P(P_), c(c_), ring(ring_), L(L_), policy(evict_first_policy()), w(threadIdx.x >> 5), lane(threadIdx.x & 31)
    {
        const int64_t r0 = share_begin(g, nw, T), r1 = share_begin(g + 1, nw, T);
        left = r1 - r0;
        if (L != nullptr) {
            // the unit holding line position r0 (the last with pre[u] <= r0)
            int lo = 0, hi = P.units - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (L->pre[mid] <= r0)
                    lo = mid;
                else
                    hi = mid - 1;
            }
            u = lo;
            j = (int)(r0 - L->pre[u]);
        } else {
            const int cap = max(P.sparse.cap, 1);
            u = (int)(r0 / cap);
            j = (int)(r0 - (int64_t)u * cap);
        }
    }

    __device__ __forceinline__ void enter(int x)
    {
        if (x != gu) {  // length and K rows of a new unit
            gu = x;
            gn = L ? span(x) : score_len(P, x, c);
            const int b = x / P.Hkv, h = x % P.Hkv;
            kbase = P.sparse.k + ((int64_t)b * P.sparse.sb + (int64_t)h * P.sparse.sh) * ES;
        }
    }

    __device__ __forceinline__ bool next(StageDesc &d)
    {
        while (left > 0) {
            enter(u);
            const int seg = (int)min(left, (int64_t)(span(u) - j));  // rows of unit u left in the share
            const int vend = min(j + seg, gn);
            if (j >= vend) {
                left -= seg;
                ++u;
                j = 0;
                continue;
            }
            const int cnt = min(Gm::SROWS, vend - j);
            const bool last = j + cnt >= vend;
            d.unit = u;
            d.start = j;
            d.count = cnt;
            d.flags = (u != last_unit ? SD_FIRST : 0) | (last ? SD_LAST : 0);
            last_unit = u;
            if (last) {
                left -= seg;
                ++u;
                j = 0;
            } else {
                left -= cnt;
                j += cnt;
            }
            return true;
        }
        return false;
    }

    // Copies of a stage (no descriptor record).
    __device__ __forceinline__ void copy_stage(const StageDesc &d, int slot)
    {
        const TierP &T = P.sparse;
        const char *src = kbase + (int64_t)d.start * T.st * ES;
        unsigned char *dst = ring.slot[w][slot];
        uint64_t *bar = &ring.full[w][slot];
        if (lane == 0) {
            mbar_arrive_expect_tx(bar, (uint32_t)(d.count * Gm::ROWB));
            if (T.st == D)
                bulk_g2s(dst, src, d.count * Gm::ROWB, bar, policy);
        }
        if (T.st != D) {
            __syncwarp();
            for (int r = lane; r < d.count; r += 32)
                bulk_g2s(dst + r * Gm::ROWB, src + (int64_t)r * T.st * ES, Gm::ROWB, bar, policy);
        }
        __syncwarp();
    }

    // A static share inside one unit, or across the end of one unit into the
    // next, whose rows are all present (the common case): the stages of its
    // one or two segments follow from their sizes alone, numbered on through
    // the warp's ring, so the warp runs this short loop instead of
    // warp_pipeline's general generator, and leaves the job at the end of its
    // static share. Returns false (having done nothing) when the share does
    // not qualify or a wait ran out.
    __device__ __forceinline__ bool run_static_share()
    {
        if (left <= 0 || P.withhold)
            return false;
        // segment 0: rows [j, j + rows0) of unit u; segment 1: rows
        // [0, rows1) of unit u + 1 (rows1 = 0: none)
        const int span0 = span(u);
        const int rows0 = (int)min(left, (int64_t)(span0 - j));
        const int rows1 = (int)(left - rows0);
        if (rows0 <= 0 || (rows1 > 0 && (u + 1 >= P.units || rows1 > span(u + 1))))
            return false;
        if (j + rows0 > (L ? span0 : score_len(P, u, c)))
            return false;
        if (rows1 > 0 && rows1 > (L ? span(u + 1) : score_len(P, u + 1, c)))
            return false;
        const auto unit_k = [&](int x) {
            const int b = x / P.Hkv, h = x % P.Hkv;
            return P.sparse.k + ((int64_t)b * P.sparse.sb + (int64_t)h * P.sparse.sh) * ES;
        };
        const char *kb0 = unit_k(u);
        const char *kb1 = rows1 > 0 ? unit_k(u + 1) : kb0;
        const int u0 = u, j0 = j;
        const int nst0 = (rows0 + Gm::SROWS - 1) / Gm::SROWS;
        const int nst = nst0 + (rows1 + Gm::SROWS - 1) / Gm::SROWS;
        const auto stage = [&](int sidx) {
            if (sidx < nst0) {
                const int st0 = j0 + sidx * Gm::SROWS;
                return StageDesc{u0, st0, min(Gm::SROWS, j0 + rows0 - st0),
                                 (sidx == 0 ? SD_FIRST : 0) | (sidx == nst0 - 1 ? SD_LAST : 0)};
            }
            const int s1 = sidx - nst0, st0 = s1 * Gm::SROWS;
            return StageDesc{u0 + 1, st0, min(Gm::SROWS, rows1 - st0),
                             (s1 == 0 ? SD_FIRST : 0) | (sidx == nst - 1 ? SD_LAST : 0)};
        };
        const auto copy = [&](int sidx, int slot) {
            kbase = sidx < nst0 ? kb0 : kb1;
            copy_stage(stage(sidx), slot);
        };
        for (int sidx = 0; sidx < NS && sidx < nst; ++sidx)
            copy(sidx, sidx);
        for (int sidx = 0; sidx < nst; ++sidx) {
            const int slot = sidx % NS;
            if (!mbar_wait(&ring.full[w][slot], (sidx / NS) & 1u, c)) {
                // let the copies already started land before returning
                for (int i = sidx; i < nst && i < sidx + NS; ++i)
                    mbar_wait_bounded(&ring.full[w][i % NS], (i / NS) & 1u, c.wait_ns);
                left = 0;
                return false;
            }
            consume(stage(sidx), ring.slot[w][slot]);
            __syncwarp();
            if (sidx + NS < nst) {
                if (lane == 0)
                    fence_proxy_async_smem();
                copy(sidx + NS, slot);
            }
        }
        gu = rows1 > 0 ? u0 + 1 : u0;
        left = 0;
        return true;
    }

    __device__ __forceinline__ void issue(const StageDesc &d, int slot)
    {
        const TierP &T = P.sparse;
        const char *src = kbase + (int64_t)d.start * T.st * ES;
        unsigned char *dst = ring.slot[w][slot];
        uint64_t *bar = &ring.full[w][slot];
        const bool arm = !P.withhold;
        if (lane == 0) {
            ring.desc[w][slot] = StageDesc{d.unit, d.start, d.count, d.flags | (arm ? SD_ARMED : 0)};
            if (arm) {
                mbar_arrive_expect_tx(bar, (uint32_t)(d.count * Gm::ROWB));
                if (T.st == D)
                    bulk_g2s(dst, src, d.count * Gm::ROWB, bar, policy);
            }
        }
        if (arm && T.st != D) {
            __syncwarp();
            for (int r = lane; r < d.count; r += 32)
                bulk_g2s(dst + r * Gm::ROWB, src + (int64_t)r * T.st * ES, Gm::ROWB, bar, policy);
        }
        __syncwarp();
    }

    __device__ __forceinline__ void consume(const StageDesc &d, const unsigned char *stage)
    {
        if (d.flags & SD_FIRST) {
            load_q<ES, D, G>(P, d.unit, lane, qv);
            tmax = -INFINITY;
            tmin = INFINITY;
        }
        const int vi = (lane % Gm::LPR) / Gm::REP;
        const bool writer = (lane % Gm::REP) == 0 && (vi % G) == 0;
        float *zu = P.z + (int64_t)d.unit * P.z_stride + d.start;
        float *lg = P.logit == nullptr
                        ? nullptr
                        : P.logit + ((int64_t)d.unit * P.sparse.cap + d.start) * logit_floats(G) + vi % G;
        const auto emit = [&](float v, int it0, bool check) {
            const int row = (it0 + vi / G) * Gm::RPW + lane / Gm::LPR;
            if (lg != nullptr && (lane % Gm::REP) == 0 && (!check || row < d.count))
                lg[row * logit_floats(G)] = v * P.scale;
#pragma unroll
            for (int o = 1; o < G; o <<= 1)
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o * Gm::REP));
            if (writer && (!check || row < d.count)) {
                const float zz = v * P.scale;
                zu[row] = zz;
                tmax = fmaxf(tmax, zz);
                if (zz != -INFINITY)
                    tmin = fminf(tmin, zz);
            }
        };
        if (d.count == Gm::SROWS) {
            // a full stage: every batch unrolled, so that the loads and products
            // of one batch overlap the reductions of the previous one
            constexpr int NBAT = Gm::SITERS / Gm::NB;
            float v[NBAT];
#pragma unroll
            for (int b = 0; b < NBAT; ++b)
                v[b] = qk_batch<ES, D, G>(stage, b * Gm::NB, lane, qv);
#pragma unroll
            for (int b = 0; b < NBAT; ++b)
                emit(v[b], b * Gm::NB, false);
        } else {
            for (int it0 = 0; it0 < Gm::SITERS && it0 * Gm::RPW < d.count; it0 += Gm::NB)
                emit(qk_batch<ES, D, G>(stage, it0, lane, qv), it0, true);
        }
        if ((d.flags & SD_LAST) && P.urange != nullptr) {
            const float mx = warp_max(tmax);
            const float mn = -warp_max(-tmin);
            if (lane == 0) {
                atomicMax(P.urange + 2 * d.unit, ord_key(mx));
                if (mn != INFINITY)
                    atomicMax(P.urange + 2 * d.unit + 1, ~ord_key(mn));
            }
        }
    }
};

// ---- attention ([TS 2.A] dense ++ selected sparse ++ condensed; [TS 2.C]
// Sparse Loading: selected rows are read through the indices) ----------------
//
// Two work lines, each split evenly over all warps of the grid:
//   line A: the dense and condensed tokens of all units (W_u + C_u per unit;
//           contiguous rows, full q.k and softmax-weighted V);
//   line B: the selected sparse tokens of all units (k_u per unit; gathered
//           rows, with the scorer's logits when hkv_step provides them).
// A line's units are laid end to end (attn_prefix: actual counts, prefix-summed
// per CTA in shared memory; else capacities, positions past a unit's tokens
// skipped), and warp g takes an equal share of it. The online-softmax state
// of a warp over its part of one unit becomes a record in slot
// line_base + g + u (unique); k_merge combines a unit's records afterwards in
// a fixed order.

template <int D, int G>
struct AttnState {
    static constexpr int NPV = D / 64;  // float2 pairs of the lane's head-dim slice (D / 32 elements)
    float m[G], l[G];
    float2 o[G][NPV > 0 ? NPV : 1];
    __device__ __forceinline__ void reset()
    {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = -INFINITY;
            l[g] = 0.f;
#pragma unroll
            for (int e = 0; e < NPV; ++e)
                o[g][e] = make_float2(0.f, 0.f);
        }
    }
};

// One attention stage: K rows at stage[0, AT_SLOT/2) (or, from_logits, the
// tokens' logit records there), V rows at stage[AT_SLOT/2, AT_SLOT).
template <int ES, int D, int G>
__device__ __forceinline__ void attn_stage(const Params &P, const unsigned char *stage, int nt, float *sc,
                                           const float2 (&qv)[G][Geo<ES, D, G>::NP], AttnState<D, G> &st,
                                           bool from_logits)
{
    using Gm = Geo<ES, D, G>;
    constexpr int NPV = AttnState<D, G>::NPV;
    const int lane = threadIdx.x & 31;
    const int vi = (lane % Gm::LPR) / Gm::REP;
    const bool writer = (lane % Gm::REP) == 0;
    const float scale2 = P.scale * LOG2E;
    // logits of the stage's tokens for all G query heads
    if (from_logits) {
        // the scorer's logits: lane r < nt converts token r's record
        if (lane < nt) {
            const float *lr = reinterpret_cast<const float *>(stage) + lane * logit_floats(G);
#pragma unroll
            for (int g = 0; g < G; ++g)
                sc[lane * G + g] = lr[g] * LOG2E;
        }
    } else if (ATTN_UNROLL_QK && nt == Gm::ATOK) {
        constexpr int NBAT = Gm::AITERS / Gm::NB;
        float v[NBAT];
#pragma unroll
        for (int b = 0; b < NBAT; ++b)
            v[b] = qk_batch<ES, D, G>(stage, b * Gm::NB, lane, qv);
#pragma unroll
        for (int b = 0; b < NBAT; ++b) {
            const int row = (b * Gm::NB + vi / G) * Gm::RPW + lane / Gm::LPR;
            if (writer)
                sc[row * G + (vi % G)] = v[b] * scale2;
        }
    } else {
        for (int it0 = 0; it0 < Gm::AITERS && it0 * Gm::RPW < nt; it0 += Gm::NB) {
            const float v = qk_batch<ES, D, G>(stage, it0, lane, qv);
            const int row = (it0 + vi / G) * Gm::RPW + lane / Gm::LPR;
            if (writer && row < nt)
                sc[row * G + (vi % G)] = v * scale2;
        }
    }
    __syncwarp();
    // online softmax: lane r owns token r of the stage (ATOK <= 32)
    float alpha[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float s_ = lane < nt ? sc[lane * G + g] : -INFINITY;
        const float mx = warp_max(s_);
        const float m_new = fmaxf(st.m[g], mx);
        alpha[g] = (m_new == -INFINITY) ? 1.0f : ex2(st.m[g] - m_new);
        const float pr = (m_new == -INFINITY || lane >= nt) ? 0.0f : ex2(s_ - m_new);
        if (lane < nt)
            sc[lane * G + g] = pr;
        st.l[g] = st.l[g] * alpha[g] + pr;  // per-lane partial, summed at the segment's end
        st.m[g] = m_new;
    }
    __syncwarp();
    // o = alpha o + sum_t p_t v_t over the lane's head-dim slice
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < NPV; ++e) {
            st.o[g][e].x *= alpha[g];
            st.o[g][e].y *= alpha[g];
        }
    const unsigned char *vbase = stage + (from_logits ? Gm::VOFF_B : AT_SLOT / 2) + lane * Gm::DPL * ES;
#pragma unroll 2
    for (int r = 0; r < nt; ++r) {
        float2 vv[NPV];
        if constexpr (ES == 2 && NPV == 2) {
            const uint2 w = *reinterpret_cast<const uint2 *>(vbase + r * Gm::ROWB);
            vv[0] = bf16x2_to_float2(w.x);
            vv[1] = bf16x2_to_float2(w.y);
        } else if constexpr (ES == 2) {
            vv[0] = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(vbase + r * Gm::ROWB));
        } else if constexpr (NPV == 2) {
            const uint4 w = *reinterpret_cast<const uint4 *>(vbase + r * Gm::ROWB);
            vv[0] = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
            vv[1] = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
        } else {
            const uint2 w = *reinterpret_cast<const uint2 *>(vbase + r * Gm::ROWB);
            vv[0] = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
        }
        float prs[G];
        if constexpr (G == 4) {
            const float4 p4 = *reinterpret_cast<const float4 *>(sc + r * 4);
            prs[0] = p4.x;
            prs[1] = p4.y;
            prs[2] = p4.z;
            prs[3] = p4.w;
        } else if constexpr (G == 2) {
            const float2 p2 = *reinterpret_cast<const float2 *>(sc + r * 2);
            prs[0] = p2.x;
            prs[1] = p2.y;
        } else {
#pragma unroll
            for (int g = 0; g < G; ++g)
                prs[g] = sc[r * G + g];
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float2 pp = make_float2(prs[g], prs[g]);
#pragma unroll
            for (int e = 0; e < NPV; ++e)
                st.o[g][e] = ffma2(pp, vv[e], st.o[g][e]);
        }
    }
    __syncwarp();
}

// Record layout (part_stride floats): o[G][D] (unnormalised, log2 domain
// weights), then m[G], then l[G]. m = -inf marks a record without tokens.

// Merge of query head g over records t_lo .. t_hi - 1 of a unit's list: its
// na line-A records in slots a0 .. a0 + na - 1, then its line-B records from
// slot b0 (fixed order), by one warp. Lane l owns head-dim elements l*DPL ..
// l*DPL + DPL - 1 of the partial (M, L, O); M = -inf when no record holds a
// token.
template <int D, int G>
__device__ void merge_records(const Params &P, int g, int a0, int na, int b0, int t_lo, int t_hi, float &M, float &L,
                              float (&O)[D / 32])
{
    constexpr int DPL = D / 32;
    constexpr int RS = part_stride(D, G);
    const int lane = threadIdx.x & 31;
    M = -INFINITY;
    L = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e)
        O[e] = 0.f;
    constexpr int RB = 8;  // records loaded together
    for (int t0 = t_lo; t0 < t_hi; t0 += RB) {
        float mt[RB], lt[RB], ot[RB][DPL];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const int t = t0 + r;
            const bool ok = t < t_hi;
            const int slot = t < na ? a0 + t : b0 + (t - na);
            const float *pr = P.part + (int64_t)(ok ? slot : 0) * RS;
            mt[r] = ok ? __ldcg(pr + G * D + g) : -INFINITY;
            lt[r] = ok ? __ldcg(pr + G * D + G + g) : 0.f;
            if constexpr (DPL == 4) {
                const float4 v = ok ? __ldcg(reinterpret_cast<const float4 *>(pr + g * D + lane * 4))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                ot[r][0] = v.x;
                ot[r][1] = v.y;
                ot[r][2] = v.z;
                ot[r][3] = v.w;
            } else {
#pragma unroll
                for (int e = 0; e < DPL; ++e)
                    ot[r][e] = ok ? __ldcg(pr + g * D + lane * DPL + e) : 0.f;
            }
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            if (mt[r] == -INFINITY)
                continue;
            const float Mn = fmaxf(M, mt[r]);
            const float a = (M == -INFINITY) ? 0.0f : ex2(M - Mn);
            const float f = ex2(mt[r] - Mn);
            L = L * a + lt[r] * f;
#pragma unroll
            for (int e = 0; e < DPL; ++e)
                O[e] = O[e] * a + ot[r][e] * f;
            M = Mn;
        }
    }
}

// Warps of the merge kernel: MERGE_SPLIT(G) warps per query head, each merging
// a contiguous part of the unit's records; the parts are then combined in order.
constexpr int MERGE_WARPS = 16;
__host__ __device__ constexpr int merge_split(int G) { return MERGE_WARPS / G; }

template <int ES, int D, int G>
struct AttnSmem {
    Ring<AT_NW, AT_SLOT, AT_STAGES> ring;
    float sc[AT_NW][SC_FLOATS];
    // attn_prefix (every line shorter than 2^31): start of each unit on line A
    // and on line B, and each unit's dense, sparse, selected and condensed counts
    int32_t pre[2][PREFIX_CAP + 1];
    int32_t uW[PREFIX_CAP], uN[PREFIX_CAP], uR[PREFIX_CAP];  // dense, sparse and rewrite-buffer rows
};

// A line of the attention work: the units' spans laid end to end and the
// share of it that this warp takes.
struct AttnLine {
    int64_t T;       // positions on the line
    int64_t NW;      // warps with a share (min(streaming warps, T)): every share is non-empty
    int64_t base;    // first record slot of the line
};

template <int ES, int D, int G>
struct AttnJob {
    using Gm = Geo<ES, D, G>;
    static constexpr int NS = AT_STAGES, NW = AT_NW;
    using SM = AttnSmem<ES, D, G>;

    const Params &P;
    const Ctl &c;
    SM &sm;
    uint64_t policy;
    int w, lane;
    AttnLine ln[2];
    int64_t g;  // this warp's index among the streaming warps
    // generator
    int line = 0;
    int64_t t = 0, t_end = 0;
    int gu = -1, gW = 0, gR = 0, gk = 0, gtot = 0, last_unit = -1;
    int64_t gS = 0, gspan = 0;
    const int32_t *gidx = nullptr;
    int gn = 0;
    // the lane's sparse index for the next stage, loaded one stage ahead
    int pf_j = 0, pf_unit = -1, pf_start = -1;
    // consumer
    float2 qv[G][Gm::NP];
    AttnState<D, G> st;
    bool had = false;
    int q_unit = -1;

    // Line A first; line B once begin_line_b gives it (the budgets it needs
    // are known only after the selection kernel).
    __device__ AttnJob(const Params &P_, const Ctl &c_, SM &sm_, const AttnLine &A, int64_t g_)
        : P(P_), c(c_), sm(sm_), policy(evict_first_policy()), w(threadIdx.x >> 5), lane(threadIdx.x & 31), g(g_)
    {
        ln[0] = A;
        ln[1] = AttnLine{0, 0, 0};
        start_line(0);
        st.reset();
    }

    __device__ __forceinline__ void begin_line_b(const AttnLine &B)
    {
        ln[1] = B;
        start_line(1);
    }

    __device__ __forceinline__ void start_line(int l)
    {
        line = l;
        gu = -1;
        last_unit = -1;
        if (g < ln[l].NW) {
            t = share_begin(g, ln[l].NW, ln[l].T);
            t_end = share_begin(g + 1, ln[l].NW, ln[l].T);
        } else {
            t = t_end = 0;
        }
    }

    // Start of unit u on the current line.
    __device__ __forceinline__ int64_t unit_start(int u) const
    {
        if (P.attn_prefix)
            return sm.pre[line][u];
        const int span = line == 0 ? P.dense.cap + P.cond.cap : min(P.bmax, P.sparse.cap);
        return (int64_t)u * span;
    }

    __device__ __forceinline__ void enter_unit(int u)
    {
        gu = u;
        gS = unit_start(u);
        gspan = unit_start(u + 1) - gS;
        int C;
        if (P.attn_prefix) {  // counts the prologue checked and kept; spans are exact
            gW = sm.uW[u];
            gn = sm.uN[u];
            gR = sm.uR[u];
            gk = sm.pre[1][u + 1] - sm.pre[1][u];
            C = sm.pre[0][u + 1] - sm.pre[0][u] - gW - gR;
        } else {
            gW = tier_len(P.dense, u, c);
            gn = tier_len(P.sparse, u, c);
            gR = 0;
            gk = unit_budget(P, u, gn, c);
            C = tier_len(P.cond, u, c);
        }
        // tokens of the unit on this line: dense ++ rewrite buffer ++ condensed
        // (A) or the selection (B)
        gtot = line == 0 ? gW + gR + C : gk;
        if (line == 1 && gk > 0)
            gidx = P.layout == HKV_LAYOUT_FLAT_SUM ? P.idx + __ldcg(P.offsets + u) : P.idx + (int64_t)u * P.bmax;
    }

    // Stages never cross a unit or a tier. Line A positions a < W are dense
    // rows, then R rows of a reused rewrite buffer, then condensed rows
    // a - W - R; line B positions are selection entries.
    __device__ __forceinline__ bool next(StageDesc &d)
    {
        for (;;) {
            if (t >= t_end)
                return false;  // the end of this line's share
            if (gu < 0 || t >= gS + gspan) {
                int u = gu + 1;
                if (gu < 0) {  // first unit of the share: binary search
                    int lo = 0, hi = P.units - 1;
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (unit_start(mid) <= t)
                            lo = mid;
                        else
                            hi = mid - 1;
                    }
                    u = lo;
                }
                while (u + 1 < P.units && unit_start(u + 1) <= t)
                    ++u;
                enter_unit(u);
            }
            const int a = (int)(t - gS);
            const int seg_end = (int)(min(t_end - gS, gspan));
            const int vend = min(seg_end, gtot);
            const int lflag = line ? SD_LINEB : 0;
            if (a >= vend) {
                // capacity partition: the share holds only unused positions of
                // this unit; one empty stage still writes the warp's record
                const bool first = gu != last_unit;
                t = gS + seg_end;
                if (!first)
                    continue;
                d = StageDesc{gu, a, 0, SD_FIRST | SD_LAST | lflag};
                last_unit = gu;
                return true;
            }
            int cnt, flags;
            if (line == 0) {
                const int tier_end = a < gW ? gW : (a < gW + gR ? gW + gR : vend);
                cnt = min(Gm::ATOK, min(vend, tier_end) - a);
                const bool contiguous = a < gW ? P.dense.st == D : (a < gW + gR ? P.rw.st == D : P.cond.st == D);
                flags = contiguous ? 0 : SD_GATHER;
            } else {
                cnt = min(P.logit != nullptr ? Gm::BTOK : Gm::ATOK, vend - a);
                flags = P.logit != nullptr ? SD_LOGIT : SD_GATHER;
            }
            const bool last = a + cnt >= vend;
            d = StageDesc{gu, a, cnt, flags | lflag | (gu != last_unit ? SD_FIRST : 0) | (last ? SD_LAST : 0)};
            last_unit = gu;
            t = last ? gS + seg_end : t + cnt;
            return true;
        }
    }

    // The tier and row of line-A position a of the current unit.
    __device__ __forceinline__ const TierP &line_a_tier(int a, int *row) const
    {
        if (a < gW) {
            *row = a;
            return P.dense;
        }
        if (a < gW + gR) {
            *row = a - gW;
            return P.rw;
        }
        *row = a - gW - gR;
        return P.cond;
    }

    // Source rows of line position a of the current unit (lane-level).
    __device__ __forceinline__ int64_t row_offset(const TierP &T_, int b, int h, int64_t r) const
    {
        return ((int64_t)b * T_.sb + (int64_t)h * T_.sh + r * T_.st) * ES;
    }

    __device__ __forceinline__ int sparse_row(const StageDesc &d) const
    {
        const int e = d.start + lane;  // selection entry
        int jj = (pf_unit == d.unit && pf_start == d.start) ? pf_j : __ldcg(gidx + e);
        if (jj < 0 || jj >= gn) {
            raise_flag(c, HKV_DEV_BAD_INDEX);
            jj = 0;
        }
        return jj;
    }

    __device__ __forceinline__ void issue(const StageDesc &d, int j)
    {
        const int u = d.unit;
        const int b = u / P.Hkv, h = u % P.Hkv;
        unsigned char *dst = sm.ring.slot[w][j];
        uint64_t *bar = &sm.ring.full[w][j];
        const bool arm = !P.withhold;
        if (lane == 0)
            sm.ring.desc[w][j] = StageDesc{d.unit, d.start, d.count, d.flags | (arm ? SD_ARMED : 0)};
        if (!arm) {
            __syncwarp();
            return;
        }
        const bool lineb = (d.flags & SD_LINEB) != 0;
        if (!lineb && !(d.flags & SD_GATHER)) {
            // contiguous dense or condensed rows: two bulk copies
            if (lane == 0) {
                mbar_arrive_expect_tx(bar, (uint32_t)(2 * d.count * Gm::ROWB));
                if (d.count > 0) {
                    int r;
                    const TierP &Tt = line_a_tier(d.start, &r);
                    const int64_t off = row_offset(Tt, b, h, r);
                    bulk_g2s(dst, Tt.k + off, d.count * Gm::ROWB, bar, policy);
                    bulk_g2s(dst + AT_SLOT / 2, Tt.v + off, d.count * Gm::ROWB, bar, policy);
                }
            }
            __syncwarp();
            return;
        }
        constexpr int LB = logit_floats(G) * 4;
        const bool from_logits = (d.flags & SD_LOGIT) != 0;
        if (from_logits) {
            // selected tokens with the scorer's logits: V rows and logit records
            // in 16-byte cp.async chunks spread over the warp (random rows
            // stream faster this way than as one bulk copy per row)
            const char *vs = nullptr, *ls = nullptr;
            int grow = 0;  // the lane's row on the V tensor map
            if (lane < d.count) {
                const int jj = sparse_row(d);
                vs = P.sparse.v + row_offset(P.sparse, b, h, jj);
                ls = reinterpret_cast<const char *>(P.logit + ((int64_t)u * P.sparse.cap + jj) * logit_floats(G));
                grow = u * P.sparse.cap + jj;
            }
            if (P.vmap_ok) {
                // the logit records by cp.async (each lane's copies counted on
                // the barrier first), then the V rows in groups of four by the
                // TMA: lane i < ng gathers rows 4i .. 4i + 3, a short last group
                // repeating its last row into the slack of the slot
                if (lane < d.count)
#pragma unroll
                    for (int i = 0; i < LB / 16; ++i)
                        cp_async16(dst + lane * LB + i * 16, ls + i * 16);
                cp_async_arrive(bar);
                __syncwarp();
                const int ng = (d.count + 3) >> 2;
                if (lane == 0)
                    mbar_arrive_expect_tx(bar, (uint32_t)(ng * 4 * Gm::ROWB));
                __syncwarp();
                int r[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    r[k] = __shfl_sync(0xffffffffu, grow, min(4 * lane + k, max(d.count - 1, 0)) & 31);
                if (lane < ng) {
                    fence_proxy_async_smem();  // this lane's copy after the warp's reads of the slot
                    tma_gather4(dst + Gm::VOFF_B + 4 * lane * Gm::ROWB, &P.vmap, r[0], r[1], r[2], r[3], bar);
                }
                __syncwarp();
                prefetch_index(d);
                return;
            }
            constexpr int CH = Gm::ROWB / 16;  // chunks of a V row
            static_assert(CH <= 32 && 32 % CH == 0, "row chunks");
            constexpr int RPI = 32 / CH;       // rows per warp instruction
            const int cc = lane % CH, rr = lane / CH;
            for (int r0 = 0; r0 < d.count; r0 += RPI) {
                const int r = r0 + rr;
                const char *v_ = reinterpret_cast<const char *>(
                    (uintptr_t)__shfl_sync(0xffffffffu, (unsigned long long)(uintptr_t)vs, r & 31));
                if (r < d.count)
                    cp_async16(dst + Gm::VOFF_B + r * Gm::ROWB + cc * 16, v_ + cc * 16);
            }
            if (lane < d.count)
#pragma unroll
                for (int i = 0; i < LB / 16; ++i)
                    cp_async16(dst + lane * LB + i * 16, ls + i * 16);
            cp_async_arrive(bar);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar);
            prefetch_index(d);
            return;
        }
        if (lineb && P.kmap_ok && P.vmap_ok) {
            // selected tokens' K and V rows in groups of four by the TMA, after
            // lane 0 has armed the slot for all of them: lane i < ng gathers
            // rows 4i .. 4i + 3 of both maps (a short last group repeats its
            // last row; a stage holds at most ATOK rows, a multiple of four)
            int grow = 0;
            if (lane < d.count)
                grow = u * P.sparse.cap + sparse_row(d);
            const int ng = (d.count + 3) >> 2;
            if (lane == 0)
                mbar_arrive_expect_tx(bar, (uint32_t)(ng * 4 * 2 * Gm::ROWB));
            __syncwarp();
            int r[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                r[k] = __shfl_sync(0xffffffffu, grow, min(4 * lane + k, max(d.count - 1, 0)) & 31);
            if (lane < ng) {
                fence_proxy_async_smem();  // this lane's copies after the warp's reads of the slot
                tma_gather4(dst + 4 * lane * Gm::ROWB, &P.kmap, r[0], r[1], r[2], r[3], bar);
                tma_gather4(dst + AT_SLOT / 2 + 4 * lane * Gm::ROWB, &P.vmap, r[0], r[1], r[2], r[3], bar);
            }
            __syncwarp();
            prefetch_index(d);
            return;
        }
        // one row per lane: K and V, one bulk copy each, after lane 0 has armed
        // the slot for all of them
        const char *ks = nullptr, *vs = nullptr;
        if (lane < d.count) {
            int64_t off;
            if (lineb) {
                const int jj = sparse_row(d);
                off = row_offset(P.sparse, b, h, jj);
                ks = P.sparse.k + off;
                vs = P.sparse.v + off;
            } else {
                int r;
                const TierP &Tt = line_a_tier(d.start + lane, &r);
                off = row_offset(Tt, b, h, r);
                ks = Tt.k + off;
                vs = Tt.v + off;
            }
        }
        const uint32_t kb = (uint32_t)Gm::ROWB;
        if (lane == 0)
            mbar_arrive_expect_tx(bar, (uint32_t)d.count * (kb + Gm::ROWB));
        __syncwarp();
        if (lane < d.count) {
            bulk_g2s(dst + lane * kb, ks, kb, bar, policy);
            bulk_g2s(dst + AT_SLOT / 2 + lane * Gm::ROWB, vs, Gm::ROWB, bar, policy);
        }
        __syncwarp();
        if (lineb)
            prefetch_index(d);
    }

    // Start loading the lane's selection entry of the stage after d (same
    // unit), to be used when that stage is issued.
    __device__ __forceinline__ void prefetch_index(const StageDesc &d)
    {
        const int ns = d.start + d.count;
        pf_unit = -1;
        if (!(d.flags & SD_LAST) && ns < gk) {
            pf_unit = d.unit;
            pf_start = ns;
            if (ns + lane < gk)
                pf_j = __ldcg(gidx + ns + lane);
        }
    }

    __device__ __forceinline__ void consume(const StageDesc &d, const unsigned char *stage)
    {
        if (d.flags & SD_FIRST) {
            st.reset();
            had = false;
        }
        if (d.count > 0) {
            if (!(d.flags & SD_LOGIT) && d.unit != q_unit) {
                load_q<ES, D, G>(P, d.unit, lane, qv);
                q_unit = d.unit;
            }
            attn_stage<ES, D, G>(P, stage, d.count, sm.sc[w], qv, st, (d.flags & SD_LOGIT) != 0);
            had = true;
        }
        if (d.flags & SD_LAST)
            finish(d);
    }

    // Write the warp's record for its part of unit d.unit on d's line.
    __device__ __forceinline__ void finish(const StageDesc &d)
    {
        constexpr int NPV = AttnState<D, G>::NPV;
        constexpr int RS = part_stride(D, G);
        const int l = (d.flags & SD_LINEB) ? 1 : 0;
        float *rec = P.part + (ln[l].base + g + d.unit) * RS;
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
            const float lsum = warp_sum(st.l[gg]);
#pragma unroll
            for (int e = 0; e < NPV; ++e)
                *reinterpret_cast<float2 *>(rec + gg * D + lane * 2 * NPV + 2 * e) = st.o[gg][e];
            if (lane == 0) {
                rec[G * D + gg] = had ? st.m[gg] : -INFINITY;
                rec[G * D + G + gg] = lsum;
            }
        }
        __syncwarp();
    }
};

// Attention prologue, part 1 (before the wait for the previous kernel): each
// thread reads the input lengths of its units (attn_prefix).
constexpr int AT_UPT = PREFIX_CAP / (AT_NW * 32);  // units per thread
struct AttnLens {
    int W[AT_UPT], N[AT_UPT], C[AT_UPT], R[AT_UPT];  // R: rows of a reused rewrite, -1 when not reused
};

__device__ __forceinline__ void attn_read_lengths(const Params &P, const Ctl &c, AttnLens &L)
{
    if (!P.attn_prefix)
        return;
#pragma unroll
    for (int i = 0; i < AT_UPT; ++i) {
        const int u = i * AT_NW * 32 + threadIdx.x;
        const bool ok = u < P.units;
        L.W[i] = ok ? tier_len(P.dense, u, c) : 0;
        L.N[i] = ok ? tier_len(P.sparse, u, c) : 0;
        L.C[i] = ok ? tier_len(P.cond, u, c) : 0;
        L.R[i] = ok && P.mti_left != nullptr && __ldcg(P.mti_left + u) > 0 ? tier_len(P.rw, u, c) : -1;
    }
}

// Part 2 (before the wait, from the inputs alone): line A -- with
// attn_prefix each unit's start on it and its dense, sparse and rewrite-buffer
// counts in shared memory.
template <int ES, int D, int G>
__device__ AttnLine attn_prologue_a(const Params &P, AttnSmem<ES, D, G> &sm, unsigned long long *red,
                                    const AttnLens &Ln)
{
    constexpr int NTA = AT_NW * 32;
    const int64_t NWt = (int64_t)gridDim.x * AT_NW;
    int64_t TA;
    if (P.attn_prefix) {
        unsigned long long ca = 0;
#pragma unroll
        for (int i = 0; i < AT_UPT; ++i) {
            if (i * NTA >= P.units)
                break;  // uniform over the CTA
            const int u = i * NTA + threadIdx.x;
            unsigned long long ta = 0;
            if (u < P.units) {
                // a unit that reuses its rewrite attends its rows on line A
                const int R = Ln.R[i] >= 0 ? Ln.R[i] : 0;
                sm.uW[u] = Ln.W[i];
                sm.uN[u] = Ln.N[i];
                sm.uR[u] = R;
                ta = (unsigned long long)(Ln.W[i] + R + Ln.C[i]);
            }
            unsigned long long sum;
            const unsigned long long ex = block_exclusive_scan<NTA>(ta, red, &sum);
            if (u < P.units)
                sm.pre[0][u] = (int32_t)(ca + ex);
            ca += sum;
        }
        if (threadIdx.x == 0)
            sm.pre[0][P.units] = (int32_t)ca;
        __syncthreads();
        TA = (int64_t)ca;
    } else {
        TA = (int64_t)P.units * (P.dense.cap + P.cond.cap);
    }
    // line A goes to the first attn_a_ctas CTAs only: with fewer units than
    // SMs those start on the SMs the selection kernel leaves free and finish
    // line A while it runs; the others start when it ends, and go straight to
    // line B
    const int64_t NWa = (int64_t)min((int)gridDim.x, max(1, P.attn_a_ctas)) * AT_NW;
    (void)NWt;
    return AttnLine{TA, min(NWa, TA), 0};
}

// Part 3 (after the wait): the budgets and line B -- with attn_prefix each
// unit's start on it; CTA 0 also writes every unit's record slots
// (rec_range[u] = first and last slot on line A, then on line B; first > last
// when empty) for k_merge.
template <int ES, int D, int G>
__device__ AttnLine attn_prologue_b(const Params &P, AttnSmem<ES, D, G> &sm, const Ctl &c, unsigned long long *red,
                                    const AttnLens &Ln, const AttnLine &A)
{
    constexpr int NTA = AT_NW * 32;
    const int64_t NWt = (int64_t)gridDim.x * AT_NW;
    int64_t TB;
    if (P.attn_prefix) {
        unsigned long long cb = 0;
#pragma unroll
        for (int i = 0; i < AT_UPT; ++i) {
            if (i * NTA >= P.units)
                break;  // uniform over the CTA
            const int u = i * NTA + threadIdx.x;
            unsigned long long tb = 0;
            if (u < P.units)  // a unit that reuses its rewrite has no selection on line B
                tb = Ln.R[i] >= 0 ? 0ull : (unsigned long long)unit_budget(P, u, Ln.N[i], c);
            unsigned long long sum;
            const unsigned long long ex = block_exclusive_scan<NTA>(tb, red, &sum);
            if (u < P.units)
                sm.pre[1][u] = (int32_t)(cb + ex);
            cb += sum;
        }
        if (threadIdx.x == 0)
            sm.pre[1][P.units] = (int32_t)cb;
        __syncthreads();
        TB = (int64_t)cb;
    } else {
        TB = (int64_t)P.units * min(P.bmax, P.sparse.cap);
    }
    const AttnLine B{TB, min(NWt, TB), NWt + P.units};
    if (blockIdx.x == 0) {
        for (int u = threadIdx.x; u < P.units; u += NTA) {
            int r[4];
            for (int l = 0; l < 2; ++l) {
                const AttnLine &L = l ? B : A;
                int64_t s0, s1;
                if (P.attn_prefix) {
                    s0 = sm.pre[l][u];
                    s1 = sm.pre[l][u + 1];
                } else {
                    const int64_t span = l ? min(P.bmax, P.sparse.cap) : P.dense.cap + P.cond.cap;
                    s0 = (int64_t)u * span;
                    s1 = s0 + span;
                }
                if (s1 > s0) {
                    r[2 * l] = (int)(L.base + share_owner(s0, L.NW, L.T) + u);
                    r[2 * l + 1] = (int)(L.base + share_owner(s1 - 1, L.NW, L.T) + u);
                } else {
                    r[2 * l] = 1;
                    r[2 * l + 1] = 0;
                }
            }
            *reinterpret_cast<int4 *>(P.rec_range + 4 * u) = make_int4(r[0], r[1], r[2], r[3]);
        }
    }
    return B;
}

// =============================================================================
// Per-unit kernels: selection, compaction, calibration (SEL_THREADS threads)
// =============================================================================

constexpr int NT = SEL_THREADS;
constexpr int SWEEP_Q = 8;  // quads per thread per batch of a score sweep

// Scores of one unit, from shared memory (ZS: staged there by stage_scores)
// or global memory, in batches of Q quads per thread with all loads in
// flight. Thread t takes quads t, t + NT, ... of each batch, whatever the
// source or its alignment, so sums taken in call order are identical on every
// path. f(z, j, valid) is called by every thread the same number of times.
template <bool ZS, typename F>
__device__ __forceinline__ void sweep_scores(const float *zu, int n, F &&f)
{
    if constexpr (ZS) {
        // staged scores: shared-memory latency is short, so a rolled loop (a
        // single copy of f's code) beats unrolling; these kernels run their
        // code once per unit and are bound by instruction fetch otherwise
        const int nq = (n + 3) >> 2;
        for (int base = 0; base < nq; base += NT * SWEEP_Q) {
#pragma unroll 1
            for (int i = 0; i < SWEEP_Q; ++i) {
                const int j = 4 * (base + i * NT + (int)threadIdx.x);
                float4 v;
                if (j + 4 <= n) {
                    v = lds4(zu + j);
                } else {
                    v.x = j < n ? lds1(zu + j) : 0.f;
                    v.y = j + 1 < n ? lds1(zu + j + 1) : 0.f;
                    v.z = j + 2 < n ? lds1(zu + j + 2) : 0.f;
                    v.w = j + 3 < n ? lds1(zu + j + 3) : 0.f;
                }
                f(v.x, j, j < n);
                f(v.y, j + 1, j + 1 < n);
                f(v.z, j + 2, j + 2 < n);
                f(v.w, j + 3, j + 3 < n);
            }
        }
        return;
    }
    constexpr int Q = SWEEP_Q;
    const bool vec = ZS || (((uintptr_t)zu) & 15) == 0;
    const int nq = (n + 3) >> 2;
    for (int base = 0; base < nq; base += NT * Q) {
        float4 v[Q];
#pragma unroll
        for (int i = 0; i < Q; ++i) {
            const int j = 4 * (base + i * NT + (int)threadIdx.x);
            if (vec && j + 4 <= n) {
                v[i] = ZS ? lds4(zu + j) : __ldcg(reinterpret_cast<const float4 *>(zu + j));
            } else {
                v[i].x = j < n ? (ZS ? lds1(zu + j) : __ldcg(zu + j)) : 0.f;
                v[i].y = j + 1 < n ? (ZS ? lds1(zu + j + 1) : __ldcg(zu + j + 1)) : 0.f;
                v[i].z = j + 2 < n ? (ZS ? lds1(zu + j + 2) : __ldcg(zu + j + 2)) : 0.f;
                v[i].w = j + 3 < n ? (ZS ? lds1(zu + j + 3) : __ldcg(zu + j + 3)) : 0.f;
            }
        }
#pragma unroll
        for (int i = 0; i < Q; ++i) {
            const int j = 4 * (base + i * NT + (int)threadIdx.x);
            f(v[i].x, j, j < n);
            f(v[i].y, j + 1, j + 1 < n);
            f(v[i].z, j + 2, j + 2 < n);
            f(v[i].w, j + 3, j + 3 < n);
        }
    }
}

// Select: linear score bins, then an exact sort of the candidates of one bin.

constexpr int SBINS = 2048;
constexpr int CAND_CAP = 6144;
constexpr int BIN_CAP = 2048;  // tokens of one bin sorted by the staged fast path

constexpr int ZSTAGE = 24576;  // scores of a unit staged in shared memory (units up to this length)

struct __align__(16) USmem {  // shared memory of the per-unit kernels
    float zs[ZSTAGE];
    uint32_t cnt[SBINS];
    unsigned long long mass[SBINS];  // bin mass (fixed point)
    unsigned long long cand[CAND_CAP];  // (order key << 32) | token index
    unsigned long long binbuf[BIN_CAP];  // the tokens of one bin, sorted (staged fast path)
    uint32_t bits[ZSTAGE / 32];          // selected tokens (staged fast path)
    unsigned long long red[NT / 32];
    float redf[NT / 32];
    int32_t bc[8];
    unsigned long long bcl[4];
    // a unit split over a cluster (select_compact_cluster): this CTA's part of
    // the bin counts, its normaliser and listed mass, tokens listed, a listing
    // overflow, tokens selected, and (rank 0) the cut every rank applies
    uint32_t cnt_part[SBINS];
    unsigned long long z_part, t_part;
    int32_t c_part, over_part, sel_part;
    int32_t pub_k, pub_kstar, pub_n_above, pub_fallback, pub_tie_last;
    uint32_t pub_key;
};

// Bin of a score: m s - z s (one fused multiply-add, with m s rounded once)
// rounded to the nearest integer, clamped to [0, SBINS - 1]; -inf and NaN land
// in the last bin. Any bin map that does not decrease as z falls serves the
// selection (the cut itself is exact), so the rounding is done with the fp32
// add of 1.5 * 2^23 (after which the float's bits are 0x4B400000 plus the
// integer) instead of conversion instructions.
struct BinFn {
    float ms, s;
    __device__ __forceinline__ int operator()(float z) const
    {
        const float t = fmaxf(fminf(fmaf(-z, s, ms), (float)(SBINS - 1)), 0.0f);
        return __float_as_int(t + 12582912.0f) - 0x4B400000;
    }
};

__device__ __forceinline__ BinFn make_bins(float m, float zlo)
{
    const float R = m - zlo;
    BinFn f;
    f.s = (R > 0.0f && isfinite(R)) ? (float)SBINS / R : 0.0f;
    f.ms = m * f.s;
    return f;
}

struct Selection {
    int32_t k, kstar;
    hkv_cut cut;
    uint32_t key;                 // order key of the cut (unused when k = 0)
    unsigned long long Zq;        // normaliser sum_j exp(beta (z_j - m)) in 40-bit fixed point
    __device__ __forceinline__ double Z() const { return (double)Zq * (1.0 / 1099511627776.0); }
};

// Top-p target in fixed point: ceil(p Z 2^40), at least 1, for Z = Zq 2^-40.
__device__ __forceinline__ unsigned long long mass_target(float p, unsigned long long Zq)
{
    const double t = ceil((double)p * (double)Zq);
    return t < 1.0 ? 1ull : (unsigned long long)t;
}

// Largest and smallest finite score of a unit.
template <bool ZS, class SM>
__device__ void unit_range(const float *zu, int n, float *m, float *zlo, SM &sm)
{
    float mx = -INFINITY, mn = INFINITY;
    sweep_scores<ZS>(zu, n, [&](float z, int, bool valid) {
        if (!valid)
            return;
        mx = fmaxf(mx, z);
        if (z != -INFINITY)
            mn = fminf(mn, z);
    });
    *m = block_max<NT>(mx, sm.redf);
    *zlo = -block_max<NT>(-mn, sm.redf);
}

// Copy a unit's n <= ZSTAGE scores into shared memory (all loads in flight);
// longer units stay in global memory. Returns whether they were staged.
template <class SM>
__device__ bool stage_scores(const float *zu, int n, SM &sm)
{
    if (n > ZSTAGE)
        return false;
    const bool vec = (((uintptr_t)zu) & 15) == 0;
    if (vec) {
        constexpr int PER = ZSTAGE / 4 / NT;
        float4 v[PER];
        const int n4 = n >> 2;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int q = i * NT + threadIdx.x;
            if (q < n4)
                v[i] = __ldcg(reinterpret_cast<const float4 *>(zu) + q);
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int q = i * NT + threadIdx.x;
            if (q < n4)
                reinterpret_cast<float4 *>(sm.zs)[q] = v[i];
        }
        for (int j = n4 * 4 + threadIdx.x; j < n; j += NT)
            sm.zs[j] = __ldcg(zu + j);
    } else {
        for (int j = threadIdx.x; j < n; j += NT)
            sm.zs[j] = __ldcg(zu + j);
    }
    __syncthreads();
    return true;
}

// Start copying a unit's first cnt <= ZSTAGE scores (zg 16-byte aligned) into
// shared memory: cp.async for the whole quads, plain loads and stores for the
// rest. The copies land after cp_async_wait_all and a barrier.
__device__ __forceinline__ void stage_scores_async(const float *zg, int cnt, float *zs)
{
    const int nq = cnt >> 2;
    for (int q = threadIdx.x; q < nq; q += NT)
        cp_async16(zs + 4 * q, zg + 4 * q);
    for (int j = 4 * nq + threadIdx.x; j < cnt; j += NT)
        zs[j] = __ldcg(zg + j);
}

// A sweep over a unit's scores in global memory that also stages them in
// shared memory: thread t takes the same quads in the same order as
// sweep_scores<true>, so sums taken in call order match it bit for bit.
template <typename F>
__device__ __forceinline__ void sweep_stage(const float *zg, float *zs, int n, F &&f)
{
    const bool vec = (((uintptr_t)zg) & 15) == 0;
    const int nq = (n + 3) >> 2;
    // a batch's loads all in flight and stored, then f over the thread's own
    // quads read back in a rolled loop (one copy of the quad's four calls of f)
    for (int base = 0; base < nq; base += NT * SWEEP_Q) {
        float4 v[SWEEP_Q];
#pragma unroll
        for (int i = 0; i < SWEEP_Q; ++i) {
            const int j = 4 * (base + i * NT + (int)threadIdx.x);
            if (vec && j + 4 <= n) {
                v[i] = __ldcg(reinterpret_cast<const float4 *>(zg + j));
            } else {
                v[i].x = j < n ? __ldcg(zg + j) : 0.f;
                v[i].y = j + 1 < n ? __ldcg(zg + j + 1) : 0.f;
                v[i].z = j + 2 < n ? __ldcg(zg + j + 2) : 0.f;
                v[i].w = j + 3 < n ? __ldcg(zg + j + 3) : 0.f;
            }
        }
#pragma unroll
        for (int i = 0; i < SWEEP_Q; ++i) {
            const int j = 4 * (base + i * NT + (int)threadIdx.x);
            if (j < n)
                reinterpret_cast<float4 *>(zs)[j >> 2] = v[i];  // j < n <= ZSTAGE, j a multiple of 4
        }
#pragma unroll 1
        for (int i = 0; i < SWEEP_Q; ++i) {
            // the quad back from shared memory (zeros past n were stored with it)
            const int j = 4 * (base + i * NT + (int)threadIdx.x);
            const float4 q4 = j < n ? lds4(zs + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            f(q4.x, j, j < n);
            f(q4.y, j + 1, j + 1 < n);
            f(q4.z, j + 2, j + 2 < n);
            f(q4.w, j + 3, j + 3 < n);
        }
    }
}

// First bin whose cumulative count (by_mass = false) or mass reaches target
// (1 <= target <= total over the bins). Returns the bin; *before_c / *before_m
// receive the count and mass of the bins before it.
template <typename MassFn>
__device__ int find_crossing(const uint32_t *cnt, MassFn mass, int nbins, bool by_mass, unsigned long long target,
                             unsigned long long *before_c, unsigned long long *before_m, USmem &sm)
{
    const int bpt = (nbins + NT - 1) / NT;
    const int lo = threadIdx.x * bpt;
    const int hi = min(nbins, lo + bpt);
    unsigned long long my_c = 0, my_m = 0;
    for (int b = lo; b < hi; ++b) {
        my_c += cnt[b];
        if (by_mass)
            my_m += mass(b);
    }
    unsigned long long tot;
    const unsigned long long ex_c = block_exclusive_scan<NT>(my_c, sm.red, &tot);
    const unsigned long long ex_m = by_mass ? block_exclusive_scan<NT>(my_m, sm.red, &tot) : 0ull;
    const unsigned long long ex = by_mass ? ex_m : ex_c;
    const unsigned long long own = by_mass ? my_m : my_c;
    if (threadIdx.x == 0) {
        sm.bc[0] = nbins - 1;
        sm.bcl[0] = 0;
        sm.bcl[1] = 0;
    }
    __syncthreads();
    if (ex < target && target <= ex + own) {
        unsigned long long cc = ex_c, mm = ex_m;
        for (int b = lo; b < hi; ++b) {
            const unsigned long long nc = cc + cnt[b];
            const unsigned long long nm = by_mass ? mm + mass(b) : 0ull;
            if ((by_mass ? nm : nc) >= target) {
                sm.bc[0] = b;
                sm.bcl[0] = cc;
                sm.bcl[1] = mm;
                break;
            }
            cc = nc;
            mm = nm;
        }
    }
    __syncthreads();
    const int b = sm.bc[0];
    *before_c = sm.bcl[0];
    *before_m = sm.bcl[1];
    __syncthreads();
    return b;
}

// Bitonic sort of cand[0, P) ascending (P a power of two).
__device__ void sort_candidates(unsigned long long *cand, int P)
{
    if (P <= 32) {
        // one warp, in registers
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            unsigned long long x = lane < P ? cand[lane] : ~0ull;
#pragma unroll 1
            for (int k = 2; k <= 32; k <<= 1)
#pragma unroll 1
                for (int j = k >> 1; j > 0; j >>= 1) {
                    const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, j);
                    const bool take_min = ((lane & j) == 0) == ((lane & k) == 0);
                    x = take_min ? (x < y ? x : y) : (x < y ? y : x);
                }
            if (lane < P)
                cand[lane] = x;
        }
        __syncthreads();
        return;
    }
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < P / 2; i += NT) {
                const int a = ((i / j) * 2 * j) + (i % j);  // lower element of the pair
                const int bix = a + j;
                const bool up = (a & k) == 0;
                const unsigned long long x = cand[a], y = cand[bix];
                if ((x > y) == up) {
                    cand[a] = y;
                    cand[bix] = x;
                }
            }
            __syncthreads();
        }
    }
}

// Append (key, index) of the lanes with `hit` to sm.cand (one shared atomic
// per warp). All lanes of the warp call it together.
__device__ __forceinline__ void gather_warp(bool hit, float z, int j, USmem &sm)
{
    const unsigned mask = __ballot_sync(0xffffffffu, hit);
    if (mask == 0)
        return;
    const int lane = threadIdx.x & 31, leader = __ffs(mask) - 1;
    int base = 0;
    if (lane == leader)
        base = satom_add(&sm.bc[1], __popc(mask));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (hit) {
        const int pos = base + __popc(mask & ((1u << lane) - 1u));
        if (pos < CAND_CAP)
            sm.cand[pos] = ((unsigned long long)score_key(z) << 32) | (uint32_t)j;
    }
}

// Collect the (key, index) of the tokens of bin `bin` into sm.cand (call only
// when the bin holds at most CAND_CAP tokens).
template <bool ZS>
__device__ void gather_bin(const float *zu, int n, const BinFn &bins, int bin, USmem &sm)
{
    if (threadIdx.x == 0)
        sm.bc[1] = 0;
    __syncthreads();
    sweep_scores<ZS>(zu, n, [&](float z, int j, bool valid) { gather_warp(valid && bins(z) == bin, z, j, sm); });
    __syncthreads();
}

// Sort the cnt_in gathered tokens of a bin by (key, index) and locate the cut:
// by_mass, the first token at which the cumulative mass (from mass_before)
// reaches `target`; else the token of rank `target` (1-based, within the bin).
// Returns its position in the sorted bin (left in buf, default sm.cand).
__device__ int sort_and_locate(int cnt_in, bool by_mass, unsigned long long target, unsigned long long mass_before,
                               float m, float bl2, USmem &sm, unsigned long long *buf = nullptr)
{
    if (buf == nullptr)
        buf = sm.cand;
    int P = 1;
    while (P < cnt_in)
        P <<= 1;
    for (int i = cnt_in + threadIdx.x; i < P; i += NT)
        buf[i] = ~0ull;
    __syncthreads();
    sort_candidates(buf, P);
    if (!by_mass)
        return (int)target - 1;
    const int per = (cnt_in + NT - 1) / NT;
    const int lo = threadIdx.x * per, hi = min(cnt_in, lo + per);
    unsigned long long mine = 0;
    for (int i = lo; i < hi; ++i)
        mine += wfix(key_score((uint32_t)(buf[i] >> 32)), m, bl2);
    unsigned long long tot;
    const unsigned long long ex = block_exclusive_scan<NT>(mine, sm.red, &tot) + mass_before;
    if (threadIdx.x == 0)
        sm.bc[2] = cnt_in - 1;
    __syncthreads();
    if (ex < target && target <= ex + mine) {
        unsigned long long acc = ex;
        for (int i = lo; i < hi; ++i) {
            acc += wfix(key_score((uint32_t)(buf[i] >> 32)), m, bl2);
            if (acc >= target) {
                sm.bc[2] = i;
                break;
            }
        }
    }
    __syncthreads();
    const int pos = sm.bc[2];
    __syncthreads();
    return pos;
}

// Exact radix descent over the 32-bit keys of the tokens of one bin (the
// fallback of sort_and_locate for bins above CAND_CAP tokens). Returns the cut
// key; *above gets the bin's tokens with a smaller key (higher score) and
// *above_mass their mass (mass targets only).
template <bool ZS>
__device__ uint32_t descend_bin(const float *zu, int n, const BinFn &bins, int bin, bool by_mass,
                                unsigned long long target, float m, float bl2, USmem &sm,
                                unsigned long long *above, unsigned long long *above_mass)
{
    // digit histograms in the candidate area, so the bin counts stay intact
    uint32_t *dcnt = reinterpret_cast<uint32_t *>(sm.cand);
    unsigned long long *dmass = sm.cand + SBINS / 2;
    static_assert(SBINS * 4 + SBINS * 8 <= sizeof(USmem::cand), "digit histograms");
    uint32_t prefix = 0;
    int shift = 32;
    unsigned long long cb = 0, mb = 0, rem = target;
    for (int lv = 0; lv < 3; ++lv) {
        const int wbits = lv < 2 ? 11 : 10;
        const int nb = 1 << wbits;
        const int pshift = shift;  // key bits at and above pshift are fixed by `prefix`
        shift -= wbits;
        for (int i = threadIdx.x; i < nb; i += NT) {
            dcnt[i] = 0;
            dmass[i] = 0;
        }
        __syncthreads();
        sweep_scores<ZS>(zu, n, [&](float z, int, bool valid) {
            if (!valid || bins(z) != bin)
                return;
            const uint32_t key = score_key(z);
            if (pshift < 32 && (key >> pshift) != prefix)
                return;
            const uint32_t d = (key >> shift) & (uint32_t)(nb - 1);
            sred_add(&dcnt[d], 1u);
            if (by_mass)
                sred_add(&dmass[d], wfix(z, m, bl2));
        });
        __syncthreads();
        unsigned long long bc_, bm_;
        const int d = find_crossing(
            dcnt, [&](int i) { return dmass[i]; }, nb, by_mass, rem, &bc_, &bm_, sm);
        cb += bc_;
        mb += bm_;
        rem -= by_mass ? bm_ : bc_;
        prefix = (prefix << wbits) | (uint32_t)d;
    }
    *above = cb;
    *above_mass = mb;
    return prefix;
}

// =============================================================================
// S2 + S3 ([TS 2.B] Logits Calibration; [Abstract], [TS 2.A] Top-p budget with
// hard limits): budget and cut of one unit, whole CTA.
//
// Scores are dropped into SBINS linear bins over [zlo, m] (the bin is a
// monotone function of the score, so bins split the descending order into
// runs). Sweep 1 counts the bins and sums the normaliser Z in double precision
// (fixed order, deterministic). The cut always lies within the first
// min(n, bmax) tokens, so sweep 2 sums the exact fixed-point mass of the bins
// up to the one holding rank bmax and gathers that bin's tokens. The bin where
// the mass reaches p Z (or where the clamped rank falls) is resolved exactly by
// sorting its tokens by (key, index); a bin too large to sort falls back to an
// exact radix descent over its keys.
// =============================================================================
template <bool ZS>
__device__ Selection select_unit(const float *zu, int n, float m, float zlo, float beta, float p, int bmin, int bmax,
                                 USmem &sm, int tb = -1)
{
    Selection r{};
    const float bl2 = beta * LOG2E;
    const BinFn bins = make_bins(m, zlo);
    for (int i = threadIdx.x; i < SBINS; i += NT) {
        sm.cnt[i] = 0;
        sm.mass[i] = 0;
    }
    __syncthreads();
    const auto mass = [&](int b) { return sm.mass[b]; };
    // sweep 1: bin counts and the normaliser (an exact sum of the fixed-point
    // weights the prefix masses add up, so it does not depend on the order)
    unsigned long long zsum = 0;
    sweep_scores<ZS>(zu, n, [&](float z, int, bool valid) {
        if (!valid)
            return;
        zsum += wfix(z, m, bl2);
        sred_add(&sm.cnt[bins(z)], 1u);
    });
    r.Zq = block_sum_u64<NT>(zsum, sm.red);
    HKV_TRACE_AT(tb < 0 ? -1 : tb + 1);

    // sweep 2: mass of the bins up to b_hi (the bin of rank min(n, bmax)) and
    // the tokens of b_hi, which hold the cut whenever the clamp at bmax decides
    const int r_hi = min(n, max(bmax, 1));
    unsigned long long hb_c = 0, hb_m = 0;
    const int b_hi = n > 0 ? find_crossing(sm.cnt, mass, SBINS, false, (unsigned long long)r_hi, &hb_c, &hb_m, sm)
                           : 0;
    HKV_TRACE_AT(tb < 0 ? -1 : tb + 7);
    const int cnt_hi = n > 0 ? (int)sm.cnt[b_hi] : 0;
    const bool gather_hi = n > 0 && cnt_hi <= CAND_CAP;
    const bool need_mass = n > 0 && p > 0.0f && p < 1.0f;
    if (threadIdx.x == 0)
        sm.bc[1] = 0;
    __syncthreads();
    if (need_mass || gather_hi) {
        sweep_scores<ZS>(zu, n, [&](float z, int j, bool valid) {
            const int bz = valid ? bins(z) : SBINS;
            if (need_mass && bz <= b_hi)
                sred_add(&sm.mass[bz], wfix(z, m, bl2));  // integer sum: exact in any order
            if (gather_hi)
                gather_warp(bz == b_hi, z, j, sm);
        });
        __syncthreads();
    }
    int gathered = gather_hi ? b_hi : -1;  // bin whose tokens sm.cand holds (unsorted)
    HKV_TRACE_AT(tb < 0 ? -1 : tb + 2);

    int kstar = -1;              // unclamped budget; -1: above bmax, not computed
    bool mass_cut = false;       // the mass search located the cut token
    bool sorted_cut = false;     // the cut token sits at cut_pos of the sorted bin in sm.cand
    int cut_pos = -1;
    unsigned long long cut_before = 0;  // tokens in the bins before the sorted bin

    if (n == 0)
        kstar = 0;
    else if (p >= 1.0f)
        kstar = n;
    else if (p <= 0.0f)
        kstar = 0;
    else {
        unsigned long long T = mass_target(p, r.Zq);
        unsigned long long part = 0;
        for (int i = threadIdx.x; i <= b_hi; i += NT)
            part += mass(i);
        const unsigned long long through = block_sum_u64<NT>(part, sm.red);
        HKV_TRACE_AT(tb < 0 ? -1 : tb + 8);
        if (through >= T) {
            unsigned long long mb_c, mb_m;
            const int b_m = find_crossing(sm.cnt, mass, SBINS, true, T, &mb_c, &mb_m, sm);
            const int cnt_in = (int)sm.cnt[b_m];
            if (cnt_in <= CAND_CAP) {
                if (gathered != b_m) {
                    gather_bin<ZS>(zu, n, bins, b_m, sm);
                    gathered = b_m;
                }
                const int pos = sort_and_locate(cnt_in, true, T, mb_m, m, bl2, sm);
                gathered = -1;  // sorted now
                kstar = (int)mb_c + pos + 1;
                sorted_cut = true;
                cut_pos = pos;
                cut_before = mb_c;
            } else {
                unsigned long long ab, am;
                const uint32_t key = descend_bin<ZS>(zu, n, bins, b_m, true, T - mb_m, m, bl2, sm, &ab, &am);
                gathered = -1;
                const unsigned long long w_at = wfix(key_score(key), m, bl2);
                const unsigned long long need = T - mb_m - am;
                kstar = (int)(mb_c + ab + (need + w_at - 1) / w_at);
                r.key = key;
                r.cut.n_above = (int32_t)(mb_c + ab);
            }
            mass_cut = true;
        }
        // else the first bmax tokens hold less than p: k* > bmax, not computed
    }
    int k = kstar < 0 ? bmax : min(kstar, bmax);
    k = max(k, bmin);
    k = min(k, n);
    r.k = k;
    r.kstar = kstar;
    if (k == 0) {
        r.key = 0;
        r.cut = hkv_cut{0.0f, 0, 0, kstar};
        __syncthreads();
        return r;
    }
    if (!(mass_cut && k == kstar)) {
        // the clamp decides: cut at rank k by count
        sorted_cut = false;
        unsigned long long kb_c, kb_m;
        const int b_k = find_crossing(sm.cnt, mass, SBINS, false, (unsigned long long)k, &kb_c, &kb_m, sm);
        HKV_TRACE_AT(tb < 0 ? -1 : tb + 9);
        const int cnt_in = (int)sm.cnt[b_k];
        if (cnt_in <= CAND_CAP) {
            if (gathered != b_k)
                gather_bin<ZS>(zu, n, bins, b_k, sm);
            cut_pos = sort_and_locate(cnt_in, false, (unsigned long long)k - kb_c, 0, m, bl2, sm);
            HKV_TRACE_AT(tb < 0 ? -1 : tb + 10);
            sorted_cut = true;
            cut_before = kb_c;
        } else {
            unsigned long long ab, am;
            r.key = descend_bin<ZS>(zu, n, bins, b_k, false, (unsigned long long)k - kb_c, m, bl2, sm, &ab, &am);
            r.cut.n_above = (int32_t)(kb_c + ab);
        }
    }
    if (sorted_cut) {
        // cut key and the tokens above it, from the sorted bin
        const uint32_t key = (uint32_t)(sm.cand[cut_pos] >> 32);
        if (threadIdx.x == 0) {
            int first = cut_pos;
            while (first > 0 && (uint32_t)(sm.cand[first - 1] >> 32) == key)
                --first;
            sm.bc[3] = first;
        }
        __syncthreads();
        r.key = key;
        r.cut.n_above = (int32_t)(cut_before + sm.bc[3]);
    }
    r.cut.z_cut = key_score(r.key);
    r.cut.n_tie = k - r.cut.n_above;
    r.cut.kstar = kstar;
    __syncthreads();
    HKV_TRACE_AT(tb < 0 ? -1 : tb + 3);
    return r;
}

// =============================================================================
// S2-S4 fused, lean, for a unit whose scores are staged in shared memory as
// the first sweep reads them (hkv_step): the same budget, cut and PAD_MAX row
// as select_unit followed by compact_unit, in three sweeps over the scores --
// (A) stage them and build the bin counts, the bins' exact fixed-point masses
// and Z; (B) gather the tokens of the few bins that can hold the cut and count,
// per warp segment, the tokens in the bins before each; (C) write the
// selection in index order -- with one scan of the bins between A and B, and
// sorts of the needed bins between B and C. Returns false, having written
// nothing, when a needed bin outgrows its buffer; the caller then takes
// select_unit and compact_unit on the staged scores.
// =============================================================================

// =============================================================================
// S2-S4 fused for a unit whose scores are staged in shared memory (hkv_step):
// the same budget and cut as select_unit followed by compact_unit, with fewer
// passes over the unit. After the count histogram (sweep 1, which also sums
// Z exactly as select_unit does), one sweep gathers every token of the bins up
// to the one holding rank min(n, bmax) -- a superset of any selection -- and
// the rest works on that short list: bin masses, the crossing bin sorted on
// its own, and a bitmap of the selected tokens expanded in index order.
// Returns false, having written nothing, when the list or a bin outgrows its
// buffer; the caller then takes select_unit and compact_unit.
// =============================================================================

// Copy the listed candidates of bin b into sm.binbuf (one pass, one shared
// atomic per warp and step: the order does not matter, the bin is sorted
// next); returns their number, or -1 when the bin holds more than BIN_CAP
// tokens.
__device__ int load_sorted_bin(int b, int ncand, const BinFn &bins, USmem &sm)
{
    const int cb = (int)sm.cnt[b];
    if (cb > BIN_CAP)
        return -1;
    if (threadIdx.x == 0)
        sm.bc[3] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    for (int base = 0; base < ncand; base += NT) {
        const int i = base + threadIdx.x;
        const unsigned long long e = i < ncand ? sm.cand[i] : 0ull;
        const bool hit = i < ncand && bins(key_score((uint32_t)(e >> 32))) == b;
        const unsigned mask = __ballot_sync(0xffffffffu, hit);
        if (mask != 0) {
            const int leader = __ffs(mask) - 1;
            int at = 0;
            if (lane == leader)
                at = satom_add(&sm.bc[3], __popc(mask));
            at = __shfl_sync(0xffffffffu, at, leader);
            if (hit)
                sm.binbuf[at + __popc(mask & ((1u << lane) - 1u))] = e;
        }
    }
    __syncthreads();
    return cb;
}

// Append the (key, index) of every staged token with bin <= b_hi to sm.cand,
// at positions from a block scan of per-thread counts (no shared counter):
// one sweep counts, the second writes. Returns the number listed.
__device__ int list_candidates(const float *zs, int n, const BinFn &bins, int b_hi, USmem &sm, int base = 0)
{
    unsigned long long mine = 0;
    sweep_scores<true>(zs, n, [&](float z, int, bool valid) { mine += (valid && bins(z) <= b_hi) ? 1u : 0u; });
    unsigned long long tot;
    int at = (int)block_exclusive_scan<NT>(mine, sm.red, &tot);
    sweep_scores<true>(zs, n, [&](float z, int j, bool valid) {
        if (valid && bins(z) <= b_hi)
            sm.cand[at++] = ((unsigned long long)score_key(z) << 32) | (uint32_t)(base + j);
    });
    __syncthreads();
    return (int)tot;
}

// One-sweep version of list_candidates: warp w walks its contiguous segment
// of the staged scores 128 tokens at a time (four per lane, a lane's tokens 32
// apart) and appends its hits to its own region of sm.cand (CAND_CAP / warps
// entries, no atomics); the regions are then closed up into one list, in
// index order. Returns the number listed, or -1 (and nothing usable in
// sm.cand) when a region overflows. Token j of zs is listed as index base + j.
__device__ int list_candidates_warp(const float *zs, int n, const BinFn &bins, int b_hi, USmem &sm, int base = 0)
{
    constexpr int NW = NT / 32, REG = CAND_CAP / NW;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int seg = ((n + NW - 1) / NW + 127) / 128 * 128;
    const int j0 = min(n, w * seg), j1 = min(n, j0 + seg);
    unsigned long long *reg = sm.cand + w * REG;
    const unsigned lower = (1u << lane) - 1u;
    int cnt = 0;
#pragma unroll 1
    for (int jb = j0; jb < j1; jb += 128) {
        float a[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = jb + 32 * e + lane;
            a[e] = j < j1 ? lds1(zs + j) : 0.f;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = jb + 32 * e + lane;
            const bool hit = j < j1 && bins(a[e]) <= b_hi;
            const unsigned m = __ballot_sync(0xffffffffu, hit);
            const int at = cnt + __popc(m & lower);
            if (hit && at < REG)
                reg[at] = ((unsigned long long)score_key(a[e]) << 32) | (uint32_t)(base + j);
            cnt += __popc(m);
        }
    }
    unsigned long long tot;
    const unsigned long long before = block_exclusive_scan<NT>(lane == 0 ? (unsigned long long)cnt : 0ull, sm.red, &tot);
    if (lane == 0)
        sm.bc[6] = 0;
    __syncthreads();
    if (lane == 0 && cnt > REG)
        sm.bc[6] = 1;
    __syncthreads();
    if (sm.bc[6] != 0) {
        __syncthreads();
        return -1;
    }
    // close up: every warp moves its region down to its place in the list; a
    // destination can overlap any earlier region, so all reads come first
    const int dst = (int)__shfl_sync(0xffffffffu, (unsigned long long)before, 0);
    constexpr int PER = (REG + 31) / 32;
    unsigned long long v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i)
        v[i] = lane + 32 * i < cnt ? reg[lane + 32 * i] : 0ull;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < PER; ++i)
        if (lane + 32 * i < cnt)
            sm.cand[dst + lane + 32 * i] = v[i];
    __syncthreads();
    return (int)tot;
}

// From the listed tokens (sm.cand[0, ncand): every token of bins 0 .. b_hi,
// b_hi the bin of rank r_hi = min(n, bmax), hb_c the tokens before it) and the
// unit's bin counts: the budget and its cut. When k > 0, *tie_last receives
// the index of the last selected token of the cut key (the selection is every
// token with a key below the cut's, and those of the cut key up to that
// index), and with `bitmap` the selected tokens are also marked in sm.bits
// (n bits, token j at bit j). Returns false when the crossing bin holds more
// than BIN_CAP tokens (the caller falls back to the general path).
__device__ bool cut_bitmap(int n, int ncand, int b_hi, unsigned long long hb_c, int r_hi, float m, float bl2,
                           const BinFn &bins, float p, int bmin, int bmax, USmem &sm, Selection &r, int tb,
                           bool bitmap, uint32_t *tie_last)
{
    const auto mass = [&](int b) { return sm.mass[b]; };
    int kstar = -1, pos = -1;
    bool mass_cut = false;
    unsigned long long before_c = 0;
    if (p >= 1.0f) {
        kstar = n;
    } else if (p <= 0.0f) {
        kstar = 0;
    } else {
        // the mass of all listed tokens first (an exact integer sum): the
        // per-bin masses are needed only when it reaches the target
        unsigned long long part = 0;
        for (int i = threadIdx.x; i < ncand; i += NT)
            part += wfix(key_score((uint32_t)(sm.cand[i] >> 32)), m, bl2);
        const unsigned long long through = block_sum_u64<NT>(part, sm.red);
        const unsigned long long T = mass_target(p, r.Zq);
        if (through >= T) {
            for (int i = threadIdx.x; i < SBINS; i += NT)
                sm.mass[i] = 0;
            __syncthreads();
            for (int i = threadIdx.x; i < ncand; i += NT) {
                const float z = key_score((uint32_t)(sm.cand[i] >> 32));
                sred_add(&sm.mass[bins(z)], wfix(z, m, bl2));
            }
            __syncthreads();
            unsigned long long mb_c, mb_m;
            const int b_m = find_crossing(sm.cnt, mass, SBINS, true, T, &mb_c, &mb_m, sm);
            const int cb = load_sorted_bin(b_m, ncand, bins, sm);
            if (cb < 0)
                return false;
            pos = sort_and_locate(cb, true, T, mb_m, m, bl2, sm, sm.binbuf);
            kstar = (int)mb_c + pos + 1;
            before_c = mb_c;
            mass_cut = true;
        }
    }
    int k = kstar < 0 ? bmax : min(kstar, bmax);
    k = min(max(k, bmin), n);
    HKV_TRACE_AT(tb < 0 ? -1 : tb + 8);
    uint32_t cut_key = 0u;
    int n_above = 0;
    if (k > 0) {
        if (!(mass_cut && k == kstar)) {
            // the clamp decides: the token of rank k (at bmax, the bin the
            // listing already found)
            unsigned long long kb_c = hb_c, kb_m = 0;
            const int b_k = k == r_hi ? b_hi
                                      : find_crossing(sm.cnt, mass, SBINS, false, (unsigned long long)k, &kb_c, &kb_m,
                                                      sm);
            HKV_TRACE_AT(tb < 0 ? -1 : tb + 9);
            const int cb = load_sorted_bin(b_k, ncand, bins, sm);
            HKV_TRACE_AT(tb < 0 ? -1 : tb + 10);
            if (cb < 0)
                return false;
            pos = sort_and_locate(cb, false, (unsigned long long)k - kb_c, 0, m, bl2, sm, sm.binbuf);
            HKV_TRACE_AT(tb < 0 ? -1 : tb + 14);
            before_c = kb_c;
        }
        cut_key = (uint32_t)(sm.binbuf[pos] >> 32);
        if (threadIdx.x == 0) {
            int first = pos;
            while (first > 0 && (uint32_t)(sm.binbuf[first - 1] >> 32) == cut_key)
                --first;
            sm.bc[4] = first;
        }
        __syncthreads();
        const int tie0 = sm.bc[4];
        n_above = (int)before_c + tie0;
        // the selected ties are the first k - n_above of the cut key in the
        // sorted bin (by index); the last of them sits at pos
        *tie_last = (uint32_t)sm.binbuf[pos];
        HKV_TRACE_AT(tb < 0 ? -1 : tb + 3);
        if (bitmap) {
            // bitmap of the selection: listed tokens above the cut, and the
            // first n_tie ties (consecutive in binbuf, by index)
            const int nwords = (n + 31) >> 5;
            for (int i = threadIdx.x; i < nwords; i += NT)
                sm.bits[i] = 0u;
            __syncthreads();
            for (int i = threadIdx.x; i < ncand; i += NT) {
                const unsigned long long e = sm.cand[i];
                if ((uint32_t)(e >> 32) < cut_key) {
                    const uint32_t j = (uint32_t)e;
                    atomicOr(&sm.bits[j >> 5], 1u << (j & 31));
                }
            }
            const int n_tie = k - n_above;
            for (int i = threadIdx.x; i < n_tie; i += NT) {
                const uint32_t j = (uint32_t)sm.binbuf[tie0 + i];
                atomicOr(&sm.bits[j >> 5], 1u << (j & 31));
            }
            __syncthreads();
        }
    }
    r.k = k;
    r.kstar = kstar;
    r.key = cut_key;
    r.cut.z_cut = key_score(cut_key);
    r.cut.n_above = n_above;
    r.cut.n_tie = k - n_above;
    r.cut.kstar = kstar;
    if (k == 0)
        r.cut = hkv_cut{0.0f, 0, 0, kstar};
    return true;
}

// The set bits of bits[w_begin, w_end) in index order, written as token
// indices (index_base + 32 w + bit) to row[at0 ...], positions below k only: thread t takes
// a contiguous run of words, a block scan gives each run its first position.
__device__ void expand_bits(const uint32_t *bits, int w_begin, int w_end, int at0, int k, int32_t *row, USmem &sm,
                            int index_base = 0)
{
    const int nw = max(0, w_end - w_begin);
    const int wpt = (nw + NT - 1) / NT;
    const int w0 = w_begin + threadIdx.x * wpt, w1 = min(w_end, w0 + wpt);
    unsigned long long cntw = 0;
    for (int i = w0; i < w1; ++i)
        cntw += __popc(bits[i]);
    unsigned long long tot;
    int at = at0 + (int)block_exclusive_scan<NT>(cntw, sm.red, &tot);
    for (int i = w0; i < w1; ++i) {
        uint32_t b = bits[i];
        while (b) {
            const int bit = __ffs(b) - 1;
            if (at < k)
                row[at] = index_base + i * 32 + bit;
            ++at;
            b &= b - 1u;
        }
    }
}

// The selected tokens of a candidate list in index order (sm.cand[0, ncand),
// as list_candidates_warp leaves it): every entry whose key is below cut_key,
// and those of cut_key with an index up to tie_last, written in list order to
// row[0, k). Warp w takes a contiguous part of the list, 32 entries a step; a
// block scan of the warps' counts places the parts.
__device__ void compact_list(int ncand, uint32_t cut_key, uint32_t tie_last, int k, int32_t *row, USmem &sm)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int seg = ((ncand + NW - 1) / NW + 31) / 32 * 32;
    const int i0 = min(ncand, w * seg), i1 = min(ncand, i0 + seg);
    const auto take = [&](int i) {
        if (i >= i1)
            return false;
        const unsigned long long e = sm.cand[i];
        const uint32_t kk = (uint32_t)(e >> 32);
        return kk < cut_key || (kk == cut_key && (uint32_t)e <= tie_last);
    };
    int cnt = 0;
#pragma unroll 1
    for (int i = i0 + lane; i - lane < i1; i += 32)
        cnt += __popc(__ballot_sync(0xffffffffu, take(i)));
    unsigned long long tot;
    const unsigned long long ex = block_exclusive_scan<NT>(lane == 0 ? (unsigned long long)cnt : 0ull, sm.red, &tot);
    int at = (int)__shfl_sync(0xffffffffu, (unsigned int)ex, 0);
    const unsigned lower = (1u << lane) - 1u;
#pragma unroll 1
    for (int i = i0 + lane; i - lane < i1; i += 32) {
        const bool t = take(i);
        const unsigned msk = __ballot_sync(0xffffffffu, t);
        const int pos = at + __popc(msk & lower);
        if (t && pos < k)
            row[pos] = (int32_t)(uint32_t)sm.cand[i];
        at += __popc(msk);
    }
}

// Selection and PAD_MAX compaction of one unit in one go, its n <= ZSTAGE
// scores staged in shared memory (zs; or staged from zg during the first sweep;
// or, zs_in_flight, still landing from this thread's cp.async copies).
// Returns false (nothing written) when a list or bin outgrows shared memory.
__device__ bool select_compact_fast(const float *zs, int n, float m, float zlo, float beta, float p, int bmin,
                                    int bmax, USmem &sm, Selection &r, int32_t *row, int pad, int tb,
                                    const float *zg = nullptr, bool zs_in_flight = false)
{
    const float bl2 = beta * LOG2E;
    const BinFn bins = make_bins(m, zlo);
    r = Selection{};
    for (int i = threadIdx.x; i < SBINS; i += NT)
        sm.cnt[i] = 0;
    if (zs_in_flight)
        cp_async_wait_all();
    __syncthreads();
    const auto mass = [&](int b) { return sm.mass[b]; };
    // sweep 1: bin counts and the normaliser (an exact sum of the fixed-point
    // weights the prefix masses add up, so it does not depend on the order),
    // staging the scores when they still are in global memory at zg
    unsigned long long zsum = 0;
    const auto count = [&](float z, int, bool valid) {
        if (!valid)
            return;
        zsum += wfix(z, m, bl2);
        sred_add(&sm.cnt[bins(z)], 1u);
    };
    if (zg != nullptr)
        sweep_stage(zg, sm.zs, n, count);
    else
        sweep_scores<true>(zs, n, count);
    r.Zq = block_sum_u64<NT>(zsum, sm.red);
    HKV_TRACE_AT(tb < 0 ? -1 : tb + 1);
    if (n > 0) {
        const int r_hi = min(n, max(bmax, 1));
        unsigned long long hb_c, hb_m;
        const int b_hi = find_crossing(sm.cnt, mass, SBINS, false, (unsigned long long)r_hi, &hb_c, &hb_m, sm);
        const int ncand = (int)hb_c + (int)sm.cnt[b_hi];
        if (ncand > CAND_CAP)
            return false;
        // the tokens of bins 0 .. b_hi: one sweep, in index order, or two
        // (in another order) when a warp's share of them outgrows its region
        const bool ordered = list_candidates_warp(zs, n, bins, b_hi, sm) >= 0;
        if (!ordered)
            list_candidates(zs, n, bins, b_hi, sm);
        HKV_TRACE_AT(tb < 0 ? -1 : tb + 2);
        uint32_t tie_last = 0;
        if (!cut_bitmap(n, ncand, b_hi, hb_c, r_hi, m, bl2, bins, p, bmin, bmax, sm, r, tb, !ordered, &tie_last))
            return false;
        if (r.k > 0 && ordered) {
            // the selected entries of the list, already in index order
            compact_list(ncand, r.key, tie_last, r.k, row, sm);
        } else if (r.k > 0) {
            // the row is built in shared memory from the bitmap (the candidate
            // list is no longer needed) and then written out with coalesced stores
            int32_t *buf = reinterpret_cast<int32_t *>(sm.cand);
            const bool in_smem = r.k <= 2 * CAND_CAP;
            expand_bits(sm.bits, 0, (n + 31) >> 5, 0, r.k, in_smem ? buf : row, sm);
            if (in_smem) {
                __syncthreads();
                for (int i = threadIdx.x; i < r.k; i += NT)
                    row[i] = buf[i];
            }
        }
    } else {
        r.cut = hkv_cut{0.0f, 0, 0, 0};
    }
    for (int i = r.k + threadIdx.x; i < pad; i += NT)
        row[i] = -1;
    __syncthreads();
    return true;
}

// Rank 0 of a cluster: every listed token of bin b, from the lists of all C
// ranks, into sm.binbuf (unordered). Returns their number, or -1 when the bin
// holds more than BIN_CAP tokens.
template <int C>
__device__ int gather_bin_cluster(int b, const BinFn &bins, USmem &sm, USmem *const (&peers)[C])
{
    const int cb = (int)sm.cnt[b];
    if (cb > BIN_CAP)
        return -1;
    if (threadIdx.x == 0)
        sm.bc[3] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
#pragma unroll 1
    for (int q = 0; q < C; ++q) {
        const USmem &src = *peers[q];
        const int cq = src.c_part;
        for (int base = 0; base < cq; base += NT) {
            const int i = base + threadIdx.x;
            const unsigned long long e = i < cq ? src.cand[i] : 0ull;
            const bool hit = i < cq && bins(key_score((uint32_t)(e >> 32))) == b;
            const unsigned mask = __ballot_sync(0xffffffffu, hit);
            if (mask != 0) {
                const int leader = __ffs(mask) - 1;
                int at = 0;
                if (lane == leader)
                    at = satom_add(&sm.bc[3], __popc(mask));
                at = __shfl_sync(0xffffffffu, at, leader);
                if (hit && at + __popc(mask & ((1u << lane) - 1u)) < BIN_CAP)
                    sm.binbuf[at + __popc(mask & ((1u << lane) - 1u))] = e;
            }
        }
    }
    __syncthreads();
    return min(sm.bc[3], cb);
}

// A unit too long to stage in one CTA, split over a cluster of C CTAs (all of
// them run this function): rank r stages tokens [r c, r c + c) of the unit's
// scores (c a multiple of 128, c <= ZSTAGE), counts and lists its part, and
// the parts meet in distributed shared memory. The cut is found by rank 0 from
// the summed bin counts and masses and the one bin that holds it, gathered from
// every rank's list; each rank then marks and expands its own part of the
// selection, after the selected tokens of the ranks before it. Every branch
// around a cluster barrier depends only on values all ranks hold alike (the
// summed counts, the published cut), so all ranks pass the same barriers, and
// the last one keeps every CTA's shared memory alive while others read it.
// Returns 0 when done (r valid on rank 0), 1 when rank 0 must redo the unit on
// the general path (a part's list or the cut's bin too large; nothing written).
template <int C>
__host__ __device__ constexpr int cluster_chunk(int n)
{
    return ((n + C - 1) / C + 127) / 128 * 128;
}

template <int C>
__device__ int select_compact_cluster(const float *zg, int n, float m, float zlo, float beta, float p, int bmin,
                                      int bmax, USmem &sm, Selection &r, int32_t *row, int pad, int tb,
                                      int rank)
{
    namespace cg = cooperative_groups;
    auto cl = cg::this_cluster();
    USmem *peers[C];
#pragma unroll
    for (int q = 0; q < C; ++q)
        peers[q] = cl.map_shared_rank(&sm, q);
    const float bl2 = beta * LOG2E;
    const BinFn bins = make_bins(m, zlo);
    const int chunk = cluster_chunk<C>(n);
    const int j0 = min(n, rank * chunk), nl = min(n, j0 + chunk) - j0;
    r = Selection{};
    for (int i = threadIdx.x; i < SBINS; i += NT)
        sm.cnt_part[i] = 0;
    __syncthreads();
    // this part's bin counts and normaliser, staging its scores
    unsigned long long zsum = 0;
    sweep_stage(zg + j0, sm.zs, nl, [&](float z, int, bool valid) {
        if (!valid)
            return;
        zsum += wfix(z, m, bl2);
        sred_add(&sm.cnt_part[bins(z)], 1u);
    });
    const unsigned long long zp = block_sum_u64<NT>(zsum, sm.red);
    if (threadIdx.x == 0)
        sm.z_part = zp;
    cl.sync();  // 1: parts counted
    for (int i = threadIdx.x; i < SBINS; i += NT) {
        uint32_t t = 0;
#pragma unroll
        for (int q = 0; q < C; ++q)
            t += peers[q]->cnt_part[i];
        sm.cnt[i] = t;
    }
#pragma unroll
    for (int q = 0; q < C; ++q)
        r.Zq += peers[q]->z_part;
    __syncthreads();
    HKV_TRACE_AT(tb < 0 ? -1 : tb + 1);
    const auto mass = [&](int b) { return sm.mass[b]; };
    const int r_hi = min(n, max(bmax, 1));
    unsigned long long hb_c, hb_m;
    const int b_hi = find_crossing(sm.cnt, mass, SBINS, false, (unsigned long long)r_hi, &hb_c, &hb_m, sm);
    // this part's tokens of bins 0 .. b_hi, and their mass
    int c = -1;
    {
        unsigned long long mine = 0;
        sweep_scores<true>(sm.zs, nl, [&](float z, int, bool valid) { mine += (valid && bins(z) <= b_hi) ? 1u : 0u; });
        unsigned long long tot;
        const int at0 = (int)block_exclusive_scan<NT>(mine, sm.red, &tot);
        if (tot <= (unsigned long long)CAND_CAP) {
            int at = at0;
            sweep_scores<true>(sm.zs, nl, [&](float z, int j, bool valid) {
                if (valid && bins(z) <= b_hi)
                    sm.cand[at++] = ((unsigned long long)score_key(z) << 32) | (uint32_t)(j0 + j);
            });
            c = (int)tot;
        }
    }
    __syncthreads();
    unsigned long long tpart = 0;
    for (int i = threadIdx.x; i < max(c, 0); i += NT)
        tpart += wfix(key_score((uint32_t)(sm.cand[i] >> 32)), m, bl2);
    tpart = block_sum_u64<NT>(tpart, sm.red);
    if (threadIdx.x == 0) {
        sm.c_part = max(c, 0);
        sm.over_part = c < 0 ? 1 : 0;
        sm.t_part = tpart;
    }
    cl.sync();  // 2: parts listed
    bool fallback = false;
    unsigned long long through = 0;
#pragma unroll
    for (int q = 0; q < C; ++q) {
        fallback |= peers[q]->over_part != 0;
        through += peers[q]->t_part;
    }
    HKV_TRACE_AT(tb < 0 ? -1 : tb + 2);
    if (!fallback) {
        const unsigned long long T = mass_target(p, r.Zq);
        const bool mass_case = p > 0.0f && p < 1.0f && through >= T;  // alike in every rank
        if (mass_case) {
            // per-bin masses of this part's listed tokens (exact integer sums)
            for (int i = threadIdx.x; i < SBINS; i += NT)
                sm.mass[i] = 0;
            __syncthreads();
            for (int i = threadIdx.x; i < sm.c_part; i += NT) {
                const float z = key_score((uint32_t)(sm.cand[i] >> 32));
                sred_add(&sm.mass[bins(z)], wfix(z, m, bl2));
            }
            __syncthreads();
            cl.sync();  // 3: part masses
        }
        if (rank == 0) {
            int kstar = p >= 1.0f ? n : (p <= 0.0f ? 0 : -1), pos = -1;
            bool mass_cut = false, bad = false;
            unsigned long long before_c = 0;
            if (mass_case) {
                for (int i = threadIdx.x; i <= b_hi; i += NT) {
                    unsigned long long t = sm.mass[i];
#pragma unroll
                    for (int q = 1; q < C; ++q)
                        t += peers[q]->mass[i];
                    sm.mass[i] = t;
                }
                __syncthreads();
                unsigned long long mb_c, mb_m;
                const int b_m = find_crossing(sm.cnt, mass, SBINS, true, T, &mb_c, &mb_m, sm);
                const int cb = gather_bin_cluster<C>(b_m, bins, sm, peers);
                if (cb < 0) {
                    bad = true;
                } else {
                    pos = sort_and_locate(cb, true, T, mb_m, m, bl2, sm, sm.binbuf);
                    kstar = (int)mb_c + pos + 1;
                    before_c = mb_c;
                    mass_cut = true;
                }
            }
            int k = kstar < 0 ? bmax : min(kstar, bmax);
            k = min(max(k, bmin), n);
            uint32_t cut_key = 0u;
            int n_above = 0, tie_last = -1;
            if (!bad && k > 0) {
                if (!(mass_cut && k == kstar)) {
                    unsigned long long kb_c = hb_c, kb_m = 0;
                    const int b_k = k == r_hi ? b_hi
                                              : find_crossing(sm.cnt, mass, SBINS, false, (unsigned long long)k,
                                                              &kb_c, &kb_m, sm);
                    const int cb = gather_bin_cluster<C>(b_k, bins, sm, peers);
                    if (cb < 0)
                        bad = true;
                    else
                        pos = sort_and_locate(cb, false, (unsigned long long)k - kb_c, 0, m, bl2, sm, sm.binbuf);
                    before_c = kb_c;
                }
                if (!bad) {
                    cut_key = (uint32_t)(sm.binbuf[pos] >> 32);
                    if (threadIdx.x == 0) {
                        int first = pos;
                        while (first > 0 && (uint32_t)(sm.binbuf[first - 1] >> 32) == cut_key)
                            --first;
                        sm.bc[4] = first;
                    }
                    __syncthreads();
                    const int tie0 = sm.bc[4];
                    n_above = (int)before_c + tie0;
                    // the selected ties are the first k - n_above by index:
                    // those up to the index of the last of them
                    tie_last = k > n_above ? (int)(uint32_t)sm.binbuf[tie0 + (k - n_above) - 1] : -1;
                }
            }
            r.k = k;
            r.kstar = kstar;
            r.key = cut_key;
            r.cut.z_cut = key_score(cut_key);
            r.cut.n_above = n_above;
            r.cut.n_tie = k - n_above;
            r.cut.kstar = kstar;
            if (k == 0)
                r.cut = hkv_cut{0.0f, 0, 0, kstar};
            if (threadIdx.x == 0) {
                sm.pub_fallback = bad ? 1 : 0;
                sm.pub_k = k;
                sm.pub_key = cut_key;
                sm.pub_tie_last = tie_last;
            }
            __syncthreads();
        }
        cl.sync();  // 4: the cut published
        const USmem &r0 = *peers[0];
        fallback = r0.pub_fallback != 0;
        const int k = r0.pub_k;
        const uint32_t key = r0.pub_key;
        const int tie_last = r0.pub_tie_last;
        if (!fallback && k > 0) {
            // this part's selected tokens as a bitmap over its own positions
            const int nwl = (nl + 31) >> 5;
            for (int i = threadIdx.x; i < nwl; i += NT)
                sm.bits[i] = 0u;
            __syncthreads();
            for (int i = threadIdx.x; i < sm.c_part; i += NT) {
                const unsigned long long e = sm.cand[i];
                const uint32_t kk = (uint32_t)(e >> 32);
                const int j = (int)(uint32_t)e;
                if (kk < key || (kk == key && j <= tie_last)) {
                    atomicOr(&sm.bits[(j - j0) >> 5], 1u << ((j - j0) & 31));
                }
            }
            __syncthreads();
            unsigned long long sc = 0;
            for (int i = threadIdx.x; i < nwl; i += NT)
                sc += __popc(sm.bits[i]);
            sc = block_sum_u64<NT>(sc, sm.red);
            if (threadIdx.x == 0)
                sm.sel_part = (int)sc;
            cl.sync();  // 5: parts' selected counts
            int at0 = 0;
            for (int q = 0; q < rank; ++q)
                at0 += peers[q]->sel_part;
            expand_bits(sm.bits, 0, nwl, at0, k, row, sm, j0);
        }
        if (rank == 0 && !fallback)
            for (int i = k + threadIdx.x; i < pad; i += NT)
                row[i] = -1;
    }
    cl.sync();  // 6: no CTA leaves while another may still read its shared memory
    return fallback ? 1 : 0;
}

// =============================================================================
// S4 Index Regularization of one unit, whole CTA ([TS 2.C] Flatten Index):
// order-preserving compaction of {key < cut key} + the first n_tie tokens with
// key == cut key into row[0, k); PAD_MAX rows are padded with -1 to `pad`.
// Warp w owns the w-th of NT/32 contiguous segments of the unit's tokens and
// walks it 32 tokens at a time (lane = token): pass 1 counts the selected and
// tied tokens with ballots, a block scan turns the counts into each warp's
// starting position and tie rank, and pass 2 writes the indices. Rolled loops
// keep the code small: the kernel runs it once per unit.
// =============================================================================
template <bool ZS>
__device__ __forceinline__ float zload(const float *zu, int j)
{
    return ZS ? lds1(zu + j) : __ldcg(zu + j);
}

template <bool ZS>
__device__ void compact_unit(const float *zu, int n, uint32_t cut_key, int n_tie, int k, int32_t *row, int pad,
                             unsigned long long *red, int tb = -1)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (k > 0) {
        const int seg = ((n + NW - 1) / NW + 31) / 32 * 32;  // tokens per warp, a multiple of 32
        const int j0 = w * seg, j1 = min(n, j0 + seg);
        // pass 1: the warp's selected (key < cut) and tied (key == cut) tokens
        uint32_t nlt = 0, neq = 0;
#pragma unroll 1
        for (int j = j0 + lane; j - lane < j1; j += 32) {
            const bool valid = j < j1;
            const uint32_t key = valid ? score_key(zload<ZS>(zu, j)) : 0xffffffffu;
            nlt += __popc(__ballot_sync(0xffffffffu, valid && key < cut_key));
            neq += __popc(__ballot_sync(0xffffffffu, valid && key == cut_key));
        }
        unsigned long long tot;
        const unsigned long long mine = lane == 0 ? (((unsigned long long)neq << 32) | nlt) : 0ull;
        const unsigned long long ex = block_exclusive_scan<NT>(mine, red, &tot);
        // every lane needs its warp's prefix: lane 0 holds it
        uint32_t lt_before = (uint32_t)__shfl_sync(0xffffffffu, (unsigned int)(ex & 0xffffffffull), 0);
        uint32_t eq_before = (uint32_t)__shfl_sync(0xffffffffu, (unsigned int)(ex >> 32), 0);
        HKV_TRACE_AT(tb < 0 ? -1 : tb + 12);
        // pass 2: positions of the taken tokens, in index order
        const unsigned lower = (1u << lane) - 1u;
#pragma unroll 1
        for (int j = j0 + lane; j - lane < j1; j += 32) {
            const bool valid = j < j1;
            const uint32_t key = valid ? score_key(zload<ZS>(zu, j)) : 0xffffffffu;
            const unsigned mlt = __ballot_sync(0xffffffffu, valid && key < cut_key);
            const unsigned meq = __ballot_sync(0xffffffffu, valid && key == cut_key);
            const uint32_t eq_rank = eq_before + __popc(meq & lower);
            const uint32_t eq_taken_before = min(eq_rank, (uint32_t)n_tie);
            const bool take = ((mlt >> lane) & 1u) || (((meq >> lane) & 1u) && eq_rank < (uint32_t)n_tie);
            const uint32_t pos = lt_before + __popc(mlt & lower) + eq_taken_before;
            if (take && pos < (uint32_t)k) {  // a caller's inconsistent cut stays in the row
                row[pos] = j;
            }
            lt_before += __popc(mlt);
            eq_before += __popc(meq);
        }
        HKV_TRACE_AT(tb < 0 ? -1 : tb + 13);
    }
    for (int i = k + threadIdx.x; i < pad; i += NT)
        row[i] = -1;
}

// =============================================================================
// Fitted temperature ([TS 2.B] calibration by temperature, [TS 3] onto the raw
// attention distribution, [TS 2.A] Tier 2 budgets from attention entropy)
//
// Per unit: the target entropy is the mean over the group's query heads of
// the entropy of each head's raw attention softmax(scale q_g . k_j) over the
// sparse tokens; the fitted inverse temperature beta in [0, FIT_BETA_MAX] is
// the root of H(beta) = target, H(beta) the entropy of softmax(beta z). H does
// not increase with beta (dH/dbeta = -beta Var(z)); the root is found by
// Newton steps kept inside a shrinking bracket (bisection when a step leaves
// it). Each unit is worked by a cluster of FIT_CTAS CTAs (one per SM), each
// taking an interleaved share of the tokens; their partial sums meet in
// distributed shared memory, added in rank order, so every CTA of the cluster
// sees the same values and takes the same branches.
// =============================================================================

constexpr float FIT_BETA_MAX = 64.0f;
constexpr int FIT_CTAS = 2;

struct __align__(16) FSmem {  // shared memory of the fitting kernel
    float zs[ZSTAGE];
    float redf[NT / 32];
    float redv[8 * (NT / 32)];
    double redd[16 * (NT / 32)];
    double xd[2][16];  // cluster exchange, two buffers used in turn
    float xf[2][8];
};

// Per-lane vectors summed (double) or maxed (float) over the CTA; every thread
// gets the result. The sums run in a fixed order.
template <int K>
__device__ __forceinline__ void block_sum_vec(double (&v)[K], double *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NW = NT / 32;
#pragma unroll
    for (int i = 0; i < K; ++i) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
        if (lane == 0)
            scratch[i * NW + warp] = v[i];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < K; ++i) {
        double r = 0.0;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            r += scratch[i * NW + w];
        v[i] = r;
    }
    __syncthreads();
}

template <int K>
__device__ __forceinline__ void block_max_vec(float (&v)[K], float *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NW = NT / 32;
#pragma unroll
    for (int i = 0; i < K; ++i) {
        v[i] = warp_max(v[i]);
        if (lane == 0)
            scratch[i * NW + warp] = v[i];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < K; ++i) {
        float r = scratch[i * NW];
#pragma unroll
        for (int w = 1; w < NW; ++w)
            r = fmaxf(r, scratch[i * NW + w]);
        v[i] = r;
    }
    __syncthreads();
}

// The cluster's CTAs combine block-uniform vectors: sums in rank order, or
// maxima. Exchanges alternate between two buffers, so one cluster barrier per
// exchange suffices: a buffer is written again only after the next barrier,
// which every CTA reaches after reading it.
struct FitCluster {
    int rank, phase;
    __device__ FitCluster() : rank((int)cooperative_groups::this_cluster().block_rank()), phase(0) {}

    template <int K>
    __device__ __forceinline__ void sum(double (&v)[K], FSmem &sm)
    {
        auto cl = cooperative_groups::this_cluster();
        double *mine = sm.xd[phase];
        if (threadIdx.x == 0) {
#pragma unroll
            for (int i = 0; i < K; ++i)
                mine[i] = v[i];
        }
        cl.sync();
#pragma unroll
        for (int i = 0; i < K; ++i) {
            double r = 0.0;
#pragma unroll
            for (int c = 0; c < FIT_CTAS; ++c)
                r += c == rank ? v[i] : cl.map_shared_rank(mine, c)[i];
            v[i] = r;
        }
        phase ^= 1;
    }

    template <int K>
    __device__ __forceinline__ void max(float (&v)[K], FSmem &sm)
    {
        auto cl = cooperative_groups::this_cluster();
        float *mine = sm.xf[phase];
        if (threadIdx.x == 0) {
#pragma unroll
            for (int i = 0; i < K; ++i)
                mine[i] = v[i];
        }
        cl.sync();
#pragma unroll
        for (int c = 0; c < FIT_CTAS; ++c) {
            if (c == rank)
                continue;
            const float *o = cl.map_shared_rank(mine, c);
#pragma unroll
            for (int i = 0; i < K; ++i)
                v[i] = fmaxf(v[i], o[i]);
        }
        phase ^= 1;
    }
};

// The G per-head logits of one record (float4 loads; LG is a multiple of 4).
template <int G>
__device__ __forceinline__ void load_record(const float *p, float (&x)[G])
{
#pragma unroll
    for (int c = 0; c < (G + 3) / 4; ++c) {
        const float4 r = __ldcg(reinterpret_cast<const float4 *>(p) + c);
        if (4 * c + 0 < G)
            x[4 * c + 0] = r.x;
        if (4 * c + 1 < G)
            x[4 * c + 1] = r.y;
        if (4 * c + 2 < G)
            x[4 * c + 2] = r.z;
        if (4 * c + 3 < G)
            x[4 * c + 3] = r.w;
    }
}

// Mean over the G heads of the entropy of softmax over a unit's n per-head
// logit records (record j at rec + j * LG, head g at offset g). The cluster's
// CTA of rank r takes records r NT + t, r NT + t + FIT_CTAS NT, ... in thread
// t. Each thread keeps per head a running maximum m, Z = sum exp(l - m) and
// S = sum exp(l - m) (l - m), rescaled when m grows (per batch of records,
// whose loads are all in flight at once); the triples are then brought to the
// cluster's maximum and summed in double. H = ln Z - S / Z.
template <int G>
__device__ float unit_attention_entropy(const float *rec, int n, FSmem &sm, FitCluster &cl)
{
    constexpr int LG = logit_floats(G);
    constexpr int BATCH = G >= 8 ? 4 : 8;
    constexpr int STRIDE = FIT_CTAS * NT;
    if (n <= 0)
        return 0.0f;
    float m[G], Z[G], S[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        Z[g] = 0.0f;
        S[g] = 0.0f;
    }
#pragma unroll 1
    for (int j0 = cl.rank * NT + threadIdx.x; j0 < n; j0 += STRIDE * BATCH) {
        float x[BATCH][G];
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            const int j = j0 + b * STRIDE;
            if (j < n) {
                load_record<G>(rec + (int64_t)j * LG, x[b]);
            } else {
#pragma unroll
                for (int g = 0; g < G; ++g)
                    x[b][g] = -INFINITY;
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float bm = x[0][g];
#pragma unroll
            for (int b = 1; b < BATCH; ++b)
                bm = fmaxf(bm, x[b][g]);
            if (bm > m[g]) {  // rescale the running sums to the new maximum
                if (Z[g] > 0.0f) {
                    const float dm = m[g] - bm;
                    const float r = ex2(dm * LOG2E);
                    S[g] = r * (S[g] + Z[g] * dm);
                    Z[g] *= r;
                }
                m[g] = bm;
            }
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                // -inf logits (and padding) weigh 0; the clamp keeps 0 * d finite
                const float d = fmaxf(x[b][g] - m[g], -FLT_MAX);
                const float e = ex2(d * LOG2E);
                Z[g] += e;
                S[g] = fmaf(e, d, S[g]);
            }
        }
    }
    float M[G];
#pragma unroll
    for (int g = 0; g < G; ++g)
        M[g] = m[g];
    block_max_vec<G>(M, sm.redv);
    cl.max<G>(M, sm);
    double acc[2 * G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        acc[2 * g] = 0.0;
        acc[2 * g + 1] = 0.0;
        if (Z[g] > 0.0f) {
            const float dm = m[g] - M[g];
            const float r = dm == 0.0f ? 1.0f : ex2(dm * LOG2E);
            acc[2 * g] = (double)(Z[g] * r);
            acc[2 * g + 1] = (double)r * ((double)S[g] + (double)Z[g] * (double)dm);
        }
    }
    block_sum_vec<2 * G>(acc, sm.redd);
    cl.sum<2 * G>(acc, sm);
    double h = 0.0;
#pragma unroll
    for (int g = 0; g < G; ++g)
        h += log(acc[2 * g]) - acc[2 * g + 1] / acc[2 * g];
    return (float)(h / G);
}

// Entropy of softmax(beta z) over a unit and its derivative in beta. The CTA of
// rank r takes the quads r NT + t, r NT + t + FIT_CTAS NT, ... in thread t and
// sums each of a quad's four positions into its own fp32 accumulators (a few
// terms each, so their rounding stays near 1e-7 relative); CTA and cluster sum
// in double.
template <bool ZS>
__device__ __forceinline__ void fit_eval(const float *zu, int n, float m, float beta, FSmem &sm, FitCluster &cl,
                                         double *H, double *dH)
{
    const float bl2 = beta * LOG2E;
    const bool vec = ZS || (((uintptr_t)zu) & 15) == 0;
    float a[4][3];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        a[i][0] = a[i][1] = a[i][2] = 0.0f;
#pragma unroll 2
    for (int j = 4 * (cl.rank * NT + (int)threadIdx.x); j < n; j += 4 * FIT_CTAS * NT) {
        float v[4];
        if (vec && j + 4 <= n) {
            const float4 t = ZS ? lds4(zu + j) : __ldcg(reinterpret_cast<const float4 *>(zu + j));
            v[0] = t.x;
            v[1] = t.y;
            v[2] = t.z;
            v[3] = t.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                v[i] = j + i < n ? (ZS ? lds1(zu + j + i) : __ldcg(zu + j + i)) : -INFINITY;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // -inf scores (and padding) weigh 0; the clamp keeps 0 * d finite
            const float d = fmaxf(v[i] - m, -FLT_MAX);
            const float w = ex2(d * bl2);
            const float wd = w * d;
            a[i][0] += w;
            a[i][1] += wd;
            a[i][2] = fmaf(wd, d, a[i][2]);
        }
    }
    double acc[3];
#pragma unroll
    for (int k = 0; k < 3; ++k)
        acc[k] = ((double)a[0][k] + (double)a[1][k]) + ((double)a[2][k] + (double)a[3][k]);
    block_sum_vec<3>(acc, sm.redd);
    cl.sum<3>(acc, sm);
    const double mean = acc[1] / acc[0];
    *H = log(acc[0]) - (double)beta * mean;
    *dH = -(double)beta * (acc[2] / acc[0] - mean * mean);
}

// The fitted inverse temperature of one unit (see the section comment). Every
// CTA of the cluster calls it with the same arguments and returns the same
// value.
template <bool ZS>
__device__ float fit_unit(const float *zu, int n, float target, FSmem &sm, FitCluster &cl, const Ctl &c, int *evals)
{
    float m, zlo;
    unit_range<ZS>(zu, n, &m, &zlo, sm);
    if (n <= 1 || !(m > zlo))
        return 1.0f;  // every beta gives the same distribution
    if (target != target) {
        if (threadIdx.x == 0 && cl.rank == 0)
            raise_flag(c, HKV_DEV_BAD_TEMP);
        return 1.0f;
    }
    const double t = (double)target;
    if (t >= log((double)n))
        return 0.0f;
    // H is known to a few 1e-7 relative (the sums' rounding), so the search
    // stops at that level: H within 2e-6 of the target, a Newton step below
    // 1e-6 of beta, or a bracket that narrow. Whether the target is reachable
    // at all (H(FIT_BETA_MAX) < target) is checked only once the search heads
    // above half of FIT_BETA_MAX.
    float lo = 0.0f, hi = FIT_BETA_MAX, beta = 1.0f;
    bool top_checked = false;
    double H, dH;
#pragma unroll 1
    for (int it = 0; it < 40; ++it) {
        fit_eval<ZS>(zu, n, m, beta, sm, cl, &H, &dH);
        ++*evals;
        if (fabs(H - t) <= 2e-6 * fmax(1.0, t))
            break;
        if (H > t)
            lo = beta;
        else
            hi = beta;
        if (hi - lo <= 1e-6f * hi)
            break;
        float next = dH < 0.0 ? (float)((double)beta - (H - t) / dH) : -1.0f;
        if (!(next > lo && next < hi))
            next = 0.5f * (lo + hi);
        else if (fabsf(next - beta) <= 1e-6f * beta)
            return next;
        if (!top_checked && next > 0.5f * FIT_BETA_MAX) {
            top_checked = true;
            double Ht, dHt;
            fit_eval<ZS>(zu, n, m, FIT_BETA_MAX, sm, cl, &Ht, &dHt);
            ++*evals;
            if (Ht >= t)
                return FIT_BETA_MAX;  // sharper than the metric can get
        }
        beta = next;
    }
    return beta;
}

}  // namespace hkv
