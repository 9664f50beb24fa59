// hkv_kernels.cuh -- device code of the HARD-KV Cascade Cache decode step.
//
// Sources: [Abstract] = arXiv abstract on the mlsanity.com page "HARD-KV:
// Head-Adaptive Regularization for Decoding-time KV Compression"; [TS 2.A],
// [TS 2.B], [TS 2.C] = sections "Cascade Cache Hierarchy", "Logits Calibration
// Mechanism", "System-Aware Index Regularization" of the gist.science Technical
// Summary of that paper.
//
// Two kinds of kernels:
//  - streaming kernels (scoring, attention): one producer warp feeds S_NCW
//    consumer warps, each through its own S_SPW-slot shared-memory ring. The
//    producer claims tiles (runs of stages) for each warp from a global ticket
//    counter and issues the stage copies (1-D TMA bulk copies for contiguous
//    rows, 16-byte cp.async for gathered rows); a stage descriptor travels with
//    the data through the slot's mbarrier. Consumers never synchronise with
//    each other, so tiles of different warps overlap freely.
//  - per-unit kernels (selection, compaction, calibration, layout): one CTA of
//    SEL_THREADS threads per (sequence, KV head).
// No tensor cores: a one-query decode is a GEMV (about 4 flop per byte), bound
// by HBM bandwidth.
#pragma once

#include "hkv_device.cuh"

namespace hkv {

constexpr int S_NCW = 8;                  // consumer warps of a streaming CTA
constexpr int S_SPW = 2;                  // ring slots per consumer warp
constexpr int S_SLOT = 8192;              // bytes per slot
constexpr int S_THREADS = (S_NCW + 1) * 32;
constexpr int S_PROD = S_NCW;             // warp index of the producer
constexpr int SCORE_TILE_STAGES = 4;      // stages per scoring tile
constexpr int ATTN_TILE_STAGES = 8;       // stages per attention tile
constexpr int SC_FLOATS = 256;            // per-warp logits of one attention stage
constexpr int TTOK_CAP = 256;             // tokens of one attention tile (any geometry)
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
    // workspace
    uint32_t *ctl;        // [0] status, [1] ticket, [2] exit count
    uint32_t *attn_done;  // [units] finished attention tiles
    float *tile_max;      // [units * score_tiles]
    float *tile_min;      // [units * score_tiles] smallest finite score of the tile
    float *part;          // [units * attn_tiles * part_stride] attention tile records
    // tiling
    int32_t score_tiles, attn_tiles;  // per unit
    int32_t score_rows;               // rows per scoring tile
    int32_t attn_toks;                // tokens per attention tile
    int32_t have_range;               // tile_max / tile_min hold the units' score range
    int32_t do_select, do_compact;    // per-unit kernel: which steps to run
    int32_t withhold;                 // fault injection: the producer never arms a slot
    uint64_t wait_ns;
};

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

// Floats of one attention tile record (o[G][D], m[G], l[G]), padded to a
// multiple of 4.
__host__ __device__ constexpr int part_stride(int D, int G) { return (G * (D + 2) + 3) / 4 * 4; }

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
    static constexpr int SITERS = S_SLOT / ITB;           // iterations per scoring stage
    static constexpr int AITERS = (S_SLOT / 2) / ITB;     // iterations over an attention stage's keys
    static constexpr int NB0 = LPR / G;
    static constexpr int NB = NB0 < AITERS ? NB0 : AITERS;  // iterations reduced together
    static constexpr int NV = NB * G;                     // partial sums per lane before reduction
    static constexpr int REP = LPR / NV;                  // lanes holding the same sum afterwards
    static constexpr int SROWS = S_SLOT / ROWB;           // rows per scoring stage
    static constexpr int ATOK = (S_SLOT / 2) / ROWB;      // tokens per attention stage
    static constexpr int DPL = D / 32;                    // PV: head-dim elements per lane
    static constexpr int QB = G * D * ES;                 // bytes of the group's queries
    static_assert(G >= 1 && G <= LPR, "group size must not exceed lanes per row");
    static_assert(ATOK * G <= SC_FLOATS && ATOK <= 32, "attention stage");
    static_assert(ATOK * ATTN_TILE_STAGES <= TTOK_CAP, "attention tile");
    static_assert(QB % 16 == 0, "query buffer");
    static_assert(SITERS % NB == 0 && AITERS % NB == 0 && LPR % NV == 0, "iteration batches");
};

// =============================================================================
// Streaming engine
// =============================================================================

enum StageKind : int32_t { STG_END = 0, STG_SCORE = 1, STG_ATTN = 2 };

struct StageDesc {
    int32_t kind, unit, start, count;  // rows (scoring) or tokens (attention) [start, start + count)
    int32_t tile, last, total, first;  // tile id; last / first stage of the tile; attention: tokens of the unit
};

struct ProdState {  // producer's view of one consumer warp
    int32_t tile, unit, next, nst, base, limit, ended, ntile;
    int32_t W, k, total, pad;
    uint32_t issued;
};

template <int ES, int D, int G>
struct __align__(128) SSmem {
    unsigned char slot[S_NCW][S_SPW][S_SLOT];
    unsigned char qbuf[S_NCW][2][G * D * ES];  // the tile's queries, double-buffered per warp
    float sc[S_NCW][SC_FLOATS];
    int32_t tidx[S_NCW][TTOK_CAP];             // producer: sparse rows of each warp's attention tile
    StageDesc desc[S_NCW][S_SPW];
    uint64_t full[S_NCW][S_SPW];
    uint64_t empty[S_NCW][S_SPW];
    ProdState ps[S_NCW];
    const char *ksrc[32], *vsrc[32];           // producer scratch: rows of one attention stage
    int32_t ticket_bc;
};

template <class SM>
__device__ __forceinline__ void stream_init(SM &sm)
{
    if (threadIdx.x == 0) {
        for (int w = 0; w < S_NCW; ++w)
            for (int j = 0; j < S_SPW; ++j) {
                mbar_init(&sm.full[w][j], 1);
                mbar_init(&sm.empty[w][j], 1);
            }
        for (int w = 0; w < S_NCW; ++w) {
            ProdState &s = sm.ps[w];
            s.tile = -1;
            s.next = s.nst = 0;
            s.ended = 0;
            s.issued = 0;
            s.ntile = 0;
            s.unit = -1;
        }
        mbar_fence_init();
    }
    __syncthreads();
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

// The lane's slice of the group's G queries (chunks l % LPR and l % LPR + LPR
// of each row), from the warp's shared query buffer.
template <int ES, int D, int G>
__device__ __forceinline__ void load_q_smem(const unsigned char *qb, int lane, float2 (&qv)[G][Geo<ES, D, G>::NP])
{
    using Gm = Geo<ES, D, G>;
    const int c0 = lane % Gm::LPR;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int cc = 0; cc < Gm::CPL; ++cc)
            unpack16<ES>(*reinterpret_cast<const uint4 *>(qb + g * Gm::ROWB + (c0 + cc * Gm::LPR) * 16),
                         &qv[g][cc * (Gm::VEC / 2)]);
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

// Is the producer's next slot of warp w free?
template <class SM>
__device__ __forceinline__ bool slot_free(SM &sm, int w)
{
    const uint32_t i = sm.ps[w].issued;
    return mbar_test(&sm.empty[w][i % S_SPW], ((i / S_SPW) & 1u) ^ 1u);
}

// Producer loop shared by both streaming kernels (all 32 lanes of the producer
// warp run it together). Tile is a policy type:
//   setup(P, sm, w, tile, c)           -- fill sm.ps[w] for a claimed tile
//   issue(P, sm, w, slot, c, policy)   -- arm the slot's barrier and copy a stage
// Returns when every consumer warp has been sent an END stage.
template <class Tile, class SM>
__device__ void producer_loop(const Params &P, SM &sm, const Ctl &c, int n_tiles, uint64_t policy)
{
    const int lane = threadIdx.x & 31;
    int rr = 0, ended = 0;
    bool exhausted = false;
    uint64_t idle_since = 0;
    while (ended < S_NCW) {
        bool want = false;
        if (lane < S_NCW && !sm.ps[lane].ended)
            want = slot_free(sm, lane);
        const unsigned mask = __ballot_sync(0xffffffffu, want);
        if (mask == 0) {
            // every ring is full: wait, bounded, for a consumer to free a slot
            if (idle_since == 0)
                idle_since = global_ns();
            else if (global_ns() - idle_since > c.wait_ns || timed_out(c)) {
                if (lane == 0)
                    raise_flag(c, HKV_DEV_TIMEOUT);
                break;
            }
            __nanosleep(64);
            continue;
        }
        idle_since = 0;
        const unsigned hi = mask & ~((1u << rr) - 1u);
        const int w = (hi ? __ffs(hi) : __ffs(mask)) - 1;
        rr = (w + 1) % S_NCW;
        ProdState &s = sm.ps[w];
        if (s.tile < 0 || s.next >= s.nst) {
            // the warp needs a new tile
            int t = n_tiles;
            if (!exhausted) {
                if (lane == 0)
                    sm.ticket_bc = (int)atomicAdd(P.ctl + 1, 1u);
                __syncwarp();
                t = sm.ticket_bc;
                __syncwarp();
            }
            if (t >= n_tiles) {
                exhausted = true;
                const uint32_t i = s.issued;
                const int j = i % S_SPW;
                if (lane == 0) {
                    sm.desc[w][j].kind = STG_END;
                    mbar_arrive(&sm.full[w][j]);
                    s.issued = i + 1;
                    s.ended = 1;
                }
                __syncwarp();
                ++ended;
                continue;
            }
            Tile::setup(P, sm, w, t, c);
            __syncwarp();
            if (s.nst == 0)
                continue;  // nothing to stream for this tile
        }
        const uint32_t i = s.issued;
        const int j = i % S_SPW;
        Tile::issue(P, sm, w, j, c, policy);
        __syncwarp();
        if (lane == 0) {
            s.issued = i + 1;
            s.next += 1;
        }
        __syncwarp();
    }
    // Before the CTA can exit, every copy this producer started must have
    // landed: wait (bounded) for the last phases it armed.
    if (lane < S_NCW) {
        const uint32_t iss = sm.ps[lane].issued;
        for (uint32_t i = iss > S_SPW ? iss - S_SPW : 0; i < iss; ++i)
            mbar_wait(&sm.full[lane][i % S_SPW], (i / S_SPW) & 1u, c);
    }
    __syncwarp();
}

// ---- scoring tiles ([TS 2.B] max-pooled attention logits; [TS 2.A] Tier 2) ----

template <int ES, int D, int G>
struct ScoreTile {
    using Gm = Geo<ES, D, G>;
    using SM = SSmem<ES, D, G>;

    __device__ static void setup(const Params &P, SM &sm, int w, int t, const Ctl &c)
    {
        const int lane = threadIdx.x & 31;
        const int u = t / P.score_tiles, ct = t % P.score_tiles;
        const int n = tier_len(P.sparse, u, c);
        const int r0 = ct * P.score_rows, r1 = min(n, r0 + P.score_rows);
        ProdState &s = sm.ps[w];
        if (lane == 0) {
            s.tile = t;
            s.unit = u;
            s.base = r0;
            s.limit = r1;
            s.next = 0;
            s.nst = r1 > r0 ? (r1 - r0 + Gm::SROWS - 1) / Gm::SROWS : 0;
            if (s.nst == 0) {  // an empty tile still reports its (empty) score range
                P.tile_max[t] = -INFINITY;
                P.tile_min[t] = INFINITY;
            }
        }
    }

    __device__ static void issue(const Params &P, SM &sm, int w, int j, const Ctl &c, uint64_t policy)
    {
        const int lane = threadIdx.x & 31;
        const ProdState &s = sm.ps[w];
        const int rs = s.base + s.next * Gm::SROWS;
        const int nr = min(Gm::SROWS, s.limit - rs);
        const int b = s.unit / P.Hkv, h = s.unit % P.Hkv;
        const TierP &T = P.sparse;
        const char *kbase = T.k + ((int64_t)b * T.sb + (int64_t)h * T.sh) * ES;
        const bool first = s.next == 0;
        const uint32_t qbytes = first ? (uint32_t)Gm::QB : 0u;
        unsigned char *qdst = sm.qbuf[w][s.ntile & 1];
        if (lane == 0) {
            StageDesc &d = sm.desc[w][j];
            d.kind = STG_SCORE;
            d.unit = s.unit;
            d.start = rs;
            d.count = nr;
            d.tile = s.tile;
            d.last = s.next == s.nst - 1;
            d.first = first;
            d.total = 0;
            if (!P.withhold) {
                mbar_arrive_expect_tx(&sm.full[w][j], (uint32_t)(nr * Gm::ROWB) + qbytes);
                if (first)
                    bulk_g2s(qdst, P.q + (int64_t)(b * P.Hq + h * G) * D * ES, Gm::QB, &sm.full[w][j], policy);
                if (T.st == D)
                    bulk_g2s(sm.slot[w][j], kbase + (int64_t)rs * T.st * ES, nr * Gm::ROWB, &sm.full[w][j],
                             policy);
            }
        }
        if (T.st != D && !P.withhold) {
            __syncwarp();
            for (int r = lane; r < nr; r += 32)
                bulk_g2s(sm.slot[w][j] + r * Gm::ROWB, kbase + (int64_t)(rs + r) * T.st * ES, Gm::ROWB,
                         &sm.full[w][j], policy);
        }
        if (lane == 0 && first)
            sm.ps[w].ntile += 1;
    }
};

// Consumer side of a scoring stage: z_j = scale * max_g q_g . k_j.
template <int ES, int D, int G>
__device__ __forceinline__ void score_stage(const Params &P, const unsigned char *stage, const StageDesc &d,
                                            const float2 (&qv)[G][Geo<ES, D, G>::NP], float &tmax, float &tmin)
{
    using Gm = Geo<ES, D, G>;
    const int lane = threadIdx.x & 31;
    const int vi = (lane % Gm::LPR) / Gm::REP;
    const bool writer = (lane % Gm::REP) == 0 && (vi % G) == 0;
    float *zu = P.z + (int64_t)d.unit * P.z_stride + d.start;
    for (int it0 = 0; it0 < Gm::SITERS && it0 * Gm::RPW < d.count; it0 += Gm::NB) {
        float v = qk_batch<ES, D, G>(stage, it0, lane, qv);
#pragma unroll
        for (int o = 1; o < G; o <<= 1)
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o * Gm::REP));
        const int row = (it0 + vi / G) * Gm::RPW + lane / Gm::LPR;
        if (writer && row < d.count) {
            const float zz = v * P.scale;
            zu[row] = zz;
            tmax = fmaxf(tmax, zz);
            if (zz != -INFINITY)
                tmin = fminf(tmin, zz);
        }
    }
}

// ---- attention tiles ([TS 2.A] dense ++ selected sparse ++ condensed;
// [TS 2.C] Sparse Loading: selected rows are read through the indices) --------

template <int ES, int D, int G>
struct AttnTile {
    using Gm = Geo<ES, D, G>;
    using SM = SSmem<ES, D, G>;

    __device__ static void setup(const Params &P, SM &sm, int w, int t, const Ctl &c)
    {
        const int lane = threadIdx.x & 31;
        const int u = t / P.attn_tiles, a = t % P.attn_tiles;
        ProdState &s = sm.ps[w];
        int W = s.W, k = s.k, total = s.total;
        if (u != s.unit) {  // lengths of a new unit (every lane loads the same words)
            const int n = tier_len(P.sparse, u, c);
            W = tier_len(P.dense, u, c);
            k = unit_budget(P, u, n, c);
            total = W + k + tier_len(P.cond, u, c);
        }
        const int t0 = a * P.attn_toks, t1 = min(total, t0 + P.attn_toks);
        // sparse rows of the tile, loaded with all loads in flight and checked
        const int s0 = max(t0, W), s1 = min(t1, W + k);
        if (s1 > s0) {
            const int32_t *idx_row =
                P.layout == HKV_LAYOUT_FLAT_SUM ? P.idx + __ldcg(P.offsets + u) : P.idx + (int64_t)u * P.bmax;
            const int n_sparse = tier_len(P.sparse, u, c);
            constexpr int PF = TTOK_CAP / 32;
            int jv[PF];
#pragma unroll
            for (int i = 0; i < PF; ++i) {
                const int tt = s0 + lane + 32 * i;
                jv[i] = tt < s1 ? __ldcg(idx_row + (tt - W)) : 0;
            }
#pragma unroll
            for (int i = 0; i < PF; ++i) {
                const int tt = s0 + lane + 32 * i;
                if (tt < s1) {
                    int jj = jv[i];
                    if (jj < 0 || jj >= n_sparse) {
                        raise_flag(c, HKV_DEV_BAD_INDEX);
                        jj = 0;
                    }
                    sm.tidx[w][tt - t0] = jj;
                }
            }
        }
        __syncwarp();
        if (lane == 0) {
            s.tile = t;
            s.unit = u;
            s.W = W;
            s.k = k;
            s.total = total;
            s.base = t0;
            s.limit = max(t0, t1);
            s.next = 0;
            // an empty tile still sends one (empty) stage so that it is counted
            s.nst = t1 > t0 ? (t1 - t0 + Gm::ATOK - 1) / Gm::ATOK : 1;
        }
    }

    __device__ static void issue(const Params &P, SM &sm, int w, int j, const Ctl &c, uint64_t policy)
    {
        const int lane = threadIdx.x & 31;
        const ProdState &s = sm.ps[w];
        const int ts = s.base + s.next * Gm::ATOK;
        const int nt = max(0, min(Gm::ATOK, s.limit - ts));
        const int b = s.unit / P.Hkv, h = s.unit % P.Hkv;
        const int W = s.W, k = s.k;
        const bool first = s.next == 0;
        unsigned char *dst = sm.slot[w][j];
        unsigned char *qdst = sm.qbuf[w][s.ntile & 1];
        const char *qsrc = P.q + (int64_t)(b * P.Hq + h * G) * D * ES;
        // contiguous dense or condensed run: two bulk copies
        const bool in_dense = ts + nt <= W && P.dense.st == D;
        const bool in_cond = ts >= W + k && P.cond.st == D;
        if (lane == 0) {
            StageDesc &d = sm.desc[w][j];
            d.kind = STG_ATTN;
            d.unit = s.unit;
            d.start = ts;
            d.count = nt;
            d.tile = s.tile;
            d.last = s.next == s.nst - 1;
            d.first = first;
            d.total = s.total;
        }
        if (!P.withhold) {
            if (nt == 0 || in_dense || in_cond) {
                if (lane == 0) {
                    const uint32_t bytes = (uint32_t)(2 * nt * Gm::ROWB) + (first ? (uint32_t)Gm::QB : 0u);
                    mbar_arrive_expect_tx(&sm.full[w][j], bytes);
                    if (first)
                        bulk_g2s(qdst, qsrc, Gm::QB, &sm.full[w][j], policy);
                    if (nt > 0) {
                        const TierP &T = in_dense ? P.dense : P.cond;
                        const int64_t r0 = in_dense ? ts : ts - W - k;
                        const int64_t off = ((int64_t)b * T.sb + (int64_t)h * T.sh + r0 * T.st) * ES;
                        bulk_g2s(dst, T.k + off, nt * Gm::ROWB, &sm.full[w][j], policy);
                        bulk_g2s(dst + S_SLOT / 2, T.v + off, nt * Gm::ROWB, &sm.full[w][j], policy);
                    }
                }
            } else {
                // gathered rows: 16-byte cp.async by the whole warp
                if (lane < nt) {
                    const int t = ts + lane;
                    const char *kb, *vb;
                    int64_t off;
                    if (t < W) {
                        kb = P.dense.k;
                        vb = P.dense.v;
                        off = (int64_t)b * P.dense.sb + (int64_t)h * P.dense.sh + (int64_t)t * P.dense.st;
                    } else if (t < W + k) {
                        kb = P.sparse.k;
                        vb = P.sparse.v;
                        off = (int64_t)b * P.sparse.sb + (int64_t)h * P.sparse.sh +
                              (int64_t)sm.tidx[w][t - s.base] * P.sparse.st;
                    } else {
                        kb = P.cond.k;
                        vb = P.cond.v;
                        off = (int64_t)b * P.cond.sb + (int64_t)h * P.cond.sh + (int64_t)(t - W - k) * P.cond.st;
                    }
                    sm.ksrc[lane] = kb + off * ES;
                    sm.vsrc[lane] = vb + off * ES;
                }
                __syncwarp();
                constexpr int CH = Gm::ROWB / 16;
                static_assert(32 % CH == 0, "row chunks");
                constexpr int RPI = 32 / CH;  // rows per warp instruction
                const int cc = lane % CH, r0 = lane / CH;
                for (int r = r0; r < nt; r += RPI) {
                    cp_async16(dst + r * Gm::ROWB + cc * 16, sm.ksrc[r] + cc * 16);
                    cp_async16(dst + S_SLOT / 2 + r * Gm::ROWB + cc * 16, sm.vsrc[r] + cc * 16);
                }
                if (first)
                    for (int i = lane; i < Gm::QB / 16; i += 32)
                        cp_async16(qdst + i * 16, qsrc + i * 16);
                cp_async_arrive(&sm.full[w][j]);
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sm.full[w][j]);
            }
        }
        if (lane == 0 && first)
            sm.ps[w].ntile += 1;
    }
};

// Online-softmax state of one warp over the tokens of its current attention
// tile, kept in the log2 domain: logits are scale * log2(e) * q . k.
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

template <int ES, int D, int G>
__device__ __forceinline__ void attn_stage(const Params &P, const unsigned char *stage, int nt, float *sc,
                                           const float2 (&qv)[G][Geo<ES, D, G>::NP], AttnState<D, G> &st)
{
    using Gm = Geo<ES, D, G>;
    constexpr int NPV = AttnState<D, G>::NPV;
    const int lane = threadIdx.x & 31;
    const int vi = (lane % Gm::LPR) / Gm::REP;
    const bool writer = (lane % Gm::REP) == 0;
    const float scale2 = P.scale * LOG2E;
    // logits of the stage's tokens for all G query heads
    for (int it0 = 0; it0 < Gm::AITERS && it0 * Gm::RPW < nt; it0 += Gm::NB) {
        const float v = qk_batch<ES, D, G>(stage, it0, lane, qv);
        const int row = (it0 + vi / G) * Gm::RPW + lane / Gm::LPR;
        if (writer && row < nt)
            sc[row * G + (vi % G)] = v * scale2;
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
        st.l[g] = st.l[g] * alpha[g] + pr;  // per-lane partial, summed at the tile's end
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
    const unsigned char *vbase = stage + S_SLOT / 2 + lane * Gm::DPL * ES;
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

// The unit's output from its attention tile records (fixed tile order), by one
// warp: lane l owns head-dim elements l*DPL .. l*DPL + DPL - 1 of every head.
template <int D, int G>
__device__ void merge_unit_warp(const Params &P, int u, int ntiles)
{
    constexpr int DPL = D / 32;
    constexpr int RS = part_stride(D, G);
    const int lane = threadIdx.x & 31;
    const int b = u / P.Hkv, h = u % P.Hkv;
    const float *rec = P.part + (int64_t)u * P.attn_tiles * RS;
    float M[G], L[G], O[G][DPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        M[g] = -INFINITY;
        L[g] = 0.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e)
            O[g][e] = 0.f;
    }
    constexpr int RB = 4;  // records loaded together
    for (int t0 = 0; t0 < ntiles; t0 += RB) {
        float mt[RB][G], lt[RB][G], ot[RB][G][DPL];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const bool ok = t0 + r < ntiles;
            const float *pr = rec + (int64_t)(t0 + r) * RS;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                mt[r][g] = ok ? __ldcg(pr + g * (D + 2) + D) : -INFINITY;
                lt[r][g] = ok ? __ldcg(pr + g * (D + 2) + D + 1) : 0.f;
#pragma unroll
                for (int e = 0; e < DPL; ++e)
                    ot[r][g][e] = ok ? __ldcg(pr + g * (D + 2) + lane * DPL + e) : 0.f;
            }
        }
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int g = 0; g < G; ++g) {
                if (mt[r][g] == -INFINITY)
                    continue;
                const float Mn = fmaxf(M[g], mt[r][g]);
                const float a = (M[g] == -INFINITY) ? 0.0f : ex2(M[g] - Mn);
                const float f = ex2(mt[r][g] - Mn);
                L[g] = L[g] * a + lt[r][g] * f;
#pragma unroll
                for (int e = 0; e < DPL; ++e)
                    O[g][e] = O[g][e] * a + ot[r][g][e] * f;
                M[g] = Mn;
            }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int hq = h * G + g;
        float *orow = P.out + ((int64_t)b * P.Hq + hq) * D + lane * DPL;
#pragma unroll
        for (int e = 0; e < DPL; ++e)
            orow[e] = (M[g] == -INFINITY) ? 0.0f : O[g][e] / L[g];
        if (lane == 0 && P.lse != nullptr)
            P.lse[(int64_t)b * P.Hq + hq] =
                (M[g] == -INFINITY) ? -INFINITY : (M[g] + log2f(L[g])) * 0.6931471805599453f;
    }
}

// Write the warp's tile record, count the tile, and merge the unit if it was
// its last tile.
template <int D, int G>
__device__ void finish_attn_tile(const Params &P, const StageDesc &d, AttnState<D, G> &st, bool had_tokens)
{
    constexpr int NPV = AttnState<D, G>::NPV;
    constexpr int RS = part_stride(D, G);
    const int lane = threadIdx.x & 31;
    const int u = d.unit, a = d.tile % P.attn_tiles;
    float lsum[G];
#pragma unroll
    for (int g = 0; g < G; ++g)
        lsum[g] = warp_sum(st.l[g]);
    if (had_tokens) {
        float *rec = P.part + ((int64_t)u * P.attn_tiles + a) * RS;
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int e = 0; e < NPV; ++e)
                *reinterpret_cast<float2 *>(rec + g * (D + 2) + lane * 2 * NPV + 2 * e) = st.o[g][e];
            if (lane == 0) {
                rec[g * (D + 2) + D] = st.m[g];
                rec[g * (D + 2) + D + 1] = lsum[g];
            }
        }
    }
    __syncwarp();
    int last = 0;
    if (lane == 0) {
        __threadfence();
        const uint32_t prev = atomicAdd(P.attn_done + u, 1u);
        last = prev == (uint32_t)P.attn_tiles - 1;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
        __threadfence();
        merge_unit_warp<D, G>(P, u, (d.total + P.attn_toks - 1) / P.attn_toks);
        if (lane == 0)
            P.attn_done[u] = 0;
    }
}

// Consumer loop of a streaming kernel: ATTN selects the attention stages
// (else scoring stages), so each kernel carries only its own consumer state.
template <int ES, int D, int G, bool ATTN>
__device__ void consumer_loop(const Params &P, SSmem<ES, D, G> &sm, const Ctl &c)
{
    using Gm = Geo<ES, D, G>;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float2 qv[G][Gm::NP];
    float tmax = -INFINITY, tmin = INFINITY;
    AttnState<D, G> st;
    if constexpr (ATTN)
        st.reset();
    bool had_tokens = false;
    uint32_t ntile = 0;
    for (uint32_t i = 0;; ++i) {
        const int j = i % S_SPW;
        if (!mbar_wait(&sm.full[w][j], (i / S_SPW) & 1u, c))
            break;
        const StageDesc d = sm.desc[w][j];
        if (d.kind == STG_END)
            break;
        if (d.first) {
            load_q_smem<ES, D, G>(sm.qbuf[w][ntile & 1], lane, qv);
            ++ntile;
        }
        const unsigned char *stage = sm.slot[w][j];
        if constexpr (!ATTN) {
            score_stage<ES, D, G>(P, stage, d, qv, tmax, tmin);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.empty[w][j]);
            if (d.last) {
                tmax = warp_max(tmax);
                tmin = -warp_max(-tmin);
                if (lane == 0) {
                    P.tile_max[d.tile] = tmax;
                    P.tile_min[d.tile] = tmin;
                }
                tmax = -INFINITY;
                tmin = INFINITY;
            }
        } else {
            if (d.count > 0) {
                attn_stage<ES, D, G>(P, stage, d.count, sm.sc[w], qv, st);
                had_tokens = true;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.empty[w][j]);
            if (d.last) {
                finish_attn_tile<D, G>(P, d, st, had_tokens);
                st.reset();
                had_tokens = false;
            }
        }
    }
}

// =============================================================================
// Per-unit kernels: selection, compaction, calibration (SEL_THREADS threads)
// =============================================================================

constexpr int NT = SEL_THREADS;

// Scores of one unit read from L2 in batches (32 per thread in flight).
// f(z, j, valid) is called by every thread the same number of times.
template <typename F>
__device__ __forceinline__ void sweep_scores(const float *zu, int n, F &&f)
{
    constexpr int BATCH = 32;
    const bool vec = (((uintptr_t)zu) & 15) == 0;
    if (vec) {
        const int n4 = n >> 2;
        const float4 *z4 = reinterpret_cast<const float4 *>(zu);
        for (int base = 0; base < n4; base += NT * (BATCH / 4)) {
            float4 v[BATCH / 4];
#pragma unroll
            for (int i = 0; i < BATCH / 4; ++i) {
                const int q4 = base + i * NT + threadIdx.x;
                v[i] = q4 < n4 ? __ldcg(z4 + q4) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int i = 0; i < BATCH / 4; ++i) {
                const int q4 = base + i * NT + threadIdx.x;
                const bool ok = q4 < n4;
                f(v[i].x, 4 * q4, ok);
                f(v[i].y, 4 * q4 + 1, ok);
                f(v[i].z, 4 * q4 + 2, ok);
                f(v[i].w, 4 * q4 + 3, ok);
            }
        }
        for (int base = n4 * 4; base < n; base += NT) {
            const int j = base + threadIdx.x;
            f(j < n ? __ldcg(zu + j) : 0.f, j, j < n);
        }
    } else {
        for (int base = 0; base < n; base += NT * BATCH) {
            float v[BATCH];
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                const int j = base + i * NT + threadIdx.x;
                v[i] = j < n ? __ldcg(zu + j) : 0.f;
            }
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                const int j = base + i * NT + threadIdx.x;
                f(v[i], j, j < n);
            }
        }
    }
}

// Select: linear score bins, then an exact sort of the candidates of one bin.
constexpr int SBINS = 2048;
constexpr int CAND_CAP = 4096;

struct __align__(16) USmem {  // shared memory of the per-unit kernels
    uint32_t cnt[SBINS];
    uint32_t mlo[SBINS];  // bin mass, low 32 bits (fixed point)
    uint32_t mhi[SBINS];  // bin mass, high 32 bits
    unsigned long long cand[CAND_CAP];  // (order key << 32) | token index
    unsigned long long red[NT / 32];
    double redd[NT / 32];
    float redf[NT / 32];
    int32_t bc[8];
    unsigned long long bcl[4];
};

// Exact 64-bit add into a (lo, hi) pair of 32-bit shared words: the carry out
// of the low word goes to the high word, so the sum is order-independent.
__device__ __forceinline__ void add_split(uint32_t *lo, uint32_t *hi, unsigned long long v)
{
    const uint32_t l = (uint32_t)v;
    const uint32_t old = atomicAdd(lo, l);
    const uint32_t h = (uint32_t)(v >> 32) + ((uint32_t)(old + l) < old ? 1u : 0u);
    if (h)
        atomicAdd(hi, h);
}

struct BinFn {
    float m, s;
    __device__ __forceinline__ int operator()(float z) const
    {
        if (z == -INFINITY)
            return SBINS - 1;
        const float t = fminf(floorf((m - z) * s), (float)(SBINS - 1));
        return (int)t;
    }
};

__device__ __forceinline__ BinFn make_bins(float m, float zlo)
{
    const float R = m - zlo;
    BinFn f;
    f.m = m;
    f.s = (R > 0.0f && isfinite(R)) ? (float)SBINS / R : 0.0f;
    return f;
}

struct Selection {
    int32_t k, kstar;
    hkv_cut cut;
    uint32_t key;                 // order key of the cut (unused when k = 0)
    double Z;                     // normaliser sum_j exp(beta (z_j - m))
};

// Largest and smallest finite score of a unit.
__device__ void unit_range(const float *zu, int n, float *m, float *zlo, USmem &sm)
{
    float mx = -INFINITY, mn = INFINITY;
    sweep_scores(zu, n, [&](float z, int, bool valid) {
        if (!valid)
            return;
        mx = fmaxf(mx, z);
        if (z != -INFINITY)
            mn = fminf(mn, z);
    });
    *m = block_max<NT>(mx, sm.redf);
    *zlo = -block_max<NT>(-mn, sm.redf);
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

__device__ __forceinline__ void gather_token(float z, int j, USmem &sm)
{
    const int pos = atomicAdd(&sm.bc[1], 1);
    if (pos < CAND_CAP)
        sm.cand[pos] = ((unsigned long long)score_key(z) << 32) | (uint32_t)j;
}

// Collect the (key, index) of the tokens of bin `bin` into sm.cand (call only
// when the bin holds at most CAND_CAP tokens).
__device__ void gather_bin(const float *zu, int n, const BinFn &bins, int bin, USmem &sm)
{
    if (threadIdx.x == 0)
        sm.bc[1] = 0;
    __syncthreads();
    sweep_scores(zu, n, [&](float z, int j, bool valid) {
        if (valid && bins(z) == bin)
            gather_token(z, j, sm);
    });
    __syncthreads();
}

// Sort the cnt_in gathered tokens of a bin by (key, index) and locate the cut:
// by_mass, the first token at which the cumulative mass (from mass_before)
// reaches `target`; else the token of rank `target` (1-based, within the bin).
// Returns its position in the sorted bin (left in sm.cand).
__device__ int sort_and_locate(int cnt_in, bool by_mass, unsigned long long target, unsigned long long mass_before,
                               float m, float bl2, USmem &sm)
{
    int P = 1;
    while (P < cnt_in)
        P <<= 1;
    for (int i = cnt_in + threadIdx.x; i < P; i += NT)
        sm.cand[i] = ~0ull;
    __syncthreads();
    sort_candidates(sm.cand, P);
    if (!by_mass)
        return (int)target - 1;
    const int per = (cnt_in + NT - 1) / NT;
    const int lo = threadIdx.x * per, hi = min(cnt_in, lo + per);
    unsigned long long mine = 0;
    for (int i = lo; i < hi; ++i)
        mine += wfix(key_score((uint32_t)(sm.cand[i] >> 32)), m, bl2);
    unsigned long long tot;
    const unsigned long long ex = block_exclusive_scan<NT>(mine, sm.red, &tot) + mass_before;
    if (threadIdx.x == 0)
        sm.bc[2] = cnt_in - 1;
    __syncthreads();
    if (ex < target && target <= ex + mine) {
        unsigned long long acc = ex;
        for (int i = lo; i < hi; ++i) {
            acc += wfix(key_score((uint32_t)(sm.cand[i] >> 32)), m, bl2);
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
        sweep_scores(zu, n, [&](float z, int, bool valid) {
            if (!valid || bins(z) != bin)
                return;
            const uint32_t key = score_key(z);
            if (pshift < 32 && (key >> pshift) != prefix)
                return;
            const uint32_t d = (key >> shift) & (uint32_t)(nb - 1);
            atomicAdd(&dcnt[d], 1u);
            if (by_mass)
                atomicAdd(&dmass[d], wfix(z, m, bl2));
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
__device__ Selection select_unit(const float *zu, int n, float m, float zlo, float beta, float p, int bmin, int bmax,
                                 USmem &sm, int tb = -1)
{
    Selection r{};
    const float bl2 = beta * LOG2E;
    const BinFn bins = make_bins(m, zlo);
    for (int i = threadIdx.x; i < SBINS; i += NT) {
        sm.cnt[i] = 0;
        sm.mlo[i] = 0;
        sm.mhi[i] = 0;
    }
    __syncthreads();
    const auto mass = [&](int b) { return ((unsigned long long)sm.mhi[b] << 32) + sm.mlo[b]; };
    // sweep 1: bin counts and the normaliser
    double zsum = 0.0;
    sweep_scores(zu, n, [&](float z, int, bool valid) {
        if (!valid)
            return;
        zsum += (double)wcal(z, m, bl2);
        atomicAdd(&sm.cnt[bins(z)], 1u);
    });
    r.Z = block_sum_f64<NT>(zsum, sm.redd);
    HKV_TRACE_AT(tb < 0 ? -1 : tb + 1);

    // sweep 2: mass of the bins up to b_hi (the bin of rank min(n, bmax)) and
    // the tokens of b_hi, which hold the cut whenever the clamp at bmax decides
    const int r_hi = min(n, max(bmax, 1));
    unsigned long long hb_c = 0, hb_m = 0;
    const int b_hi = n > 0 ? find_crossing(sm.cnt, mass, SBINS, false, (unsigned long long)r_hi, &hb_c, &hb_m, sm)
                           : 0;
    const int cnt_hi = n > 0 ? (int)sm.cnt[b_hi] : 0;
    const bool gather_hi = n > 0 && cnt_hi <= CAND_CAP;
    const bool need_mass = n > 0 && p > 0.0f && p < 1.0f;
    if (threadIdx.x == 0)
        sm.bc[1] = 0;
    __syncthreads();
    if (need_mass || gather_hi) {
        sweep_scores(zu, n, [&](float z, int j, bool valid) {
            const int bz = valid ? bins(z) : SBINS;
            if (need_mass && bz <= b_hi)
                add_split(&sm.mlo[bz], &sm.mhi[bz], wfix(z, m, bl2));
            if (gather_hi && bz == b_hi)
                gather_token(z, j, sm);
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
        const double t = ceil((double)p * r.Z * 1099511627776.0);
        unsigned long long T = t < 1.0 ? 1ull : (unsigned long long)t;
        unsigned long long part = 0;
        for (int i = threadIdx.x; i <= b_hi; i += NT)
            part += mass(i);
        const unsigned long long through = block_sum_u64<NT>(part, sm.red);
        if (through >= T) {
            unsigned long long mb_c, mb_m;
            const int b_m = find_crossing(sm.cnt, mass, SBINS, true, T, &mb_c, &mb_m, sm);
            const int cnt_in = (int)sm.cnt[b_m];
            if (cnt_in <= CAND_CAP) {
                if (gathered != b_m) {
                    gather_bin(zu, n, bins, b_m, sm);
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
                const uint32_t key = descend_bin(zu, n, bins, b_m, true, T - mb_m, m, bl2, sm, &ab, &am);
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
        const int cnt_in = (int)sm.cnt[b_k];
        if (cnt_in <= CAND_CAP) {
            if (gathered != b_k)
                gather_bin(zu, n, bins, b_k, sm);
            cut_pos = sort_and_locate(cnt_in, false, (unsigned long long)k - kb_c, 0, m, bl2, sm);
            sorted_cut = true;
            cut_before = kb_c;
        } else {
            unsigned long long ab, am;
            r.key = descend_bin(zu, n, bins, b_k, false, (unsigned long long)k - kb_c, m, bl2, sm, &ab, &am);
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
// S4 Index Regularization of one unit, whole CTA ([TS 2.C] Flatten Index):
// order-preserving compaction of {key < cut key} + the first n_tie tokens with
// key == cut key into row[0, k); PAD_MAX rows are padded with -1 to `pad`.
// Each thread takes E consecutive tokens of a chunk (loaded together).
// =============================================================================
__device__ void compact_unit(const float *zu, int n, uint32_t cut_key, int n_tie, int k, int32_t *row, int pad,
                             unsigned long long *red)
{
    constexpr int E = 16;
    unsigned long long lt_carry = 0, eq_carry = 0;
    const bool vec = (((uintptr_t)zu) & 15) == 0;
    if (k > 0) {
        for (int base = 0; base < n; base += NT * E) {
            const int j0 = base + threadIdx.x * E;
            float zz[E];
            if (vec && j0 + E <= n) {
#pragma unroll
                for (int e = 0; e < E; e += 4) {
                    const float4 v = __ldcg(reinterpret_cast<const float4 *>(zu + j0 + e));
                    zz[e] = v.x;
                    zz[e + 1] = v.y;
                    zz[e + 2] = v.z;
                    zz[e + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e)
                    zz[e] = (j0 + e < n) ? __ldcg(zu + j0 + e) : 0.f;
            }
            uint32_t lt_bits = 0, eq_bits = 0;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const uint32_t key = score_key(zz[e]);
                const bool valid = j0 + e < n;
                lt_bits |= (valid && key < cut_key) ? (1u << e) : 0u;
                eq_bits |= (valid && key == cut_key) ? (1u << e) : 0u;
            }
            const uint32_t nlt = __popc(lt_bits), neq = __popc(eq_bits);
            unsigned long long tot;
            const unsigned long long ex =
                block_exclusive_scan<NT>(((unsigned long long)neq << 32) | nlt, red, &tot);
            const unsigned long long eq_before = eq_carry + (ex >> 32);
            const unsigned long long lt_before = lt_carry + (ex & 0xffffffffull);
            unsigned long long pos = lt_before + min(eq_before, (unsigned long long)n_tie);
            unsigned long long eq_rank = eq_before;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                bool take = (lt_bits >> e) & 1u;
                if ((eq_bits >> e) & 1u) {
                    take = eq_rank < (unsigned long long)n_tie;
                    ++eq_rank;
                }
                if (take && pos < (unsigned long long)k)  // a caller's inconsistent cut stays in the row
                    row[pos++] = j0 + e;
            }
            lt_carry += tot & 0xffffffffull;
            eq_carry += tot >> 32;
        }
    }
    for (int i = k + threadIdx.x; i < pad; i += NT)
        row[i] = -1;
}

}  // namespace hkv
