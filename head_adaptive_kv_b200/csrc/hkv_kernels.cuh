// hkv_kernels.cuh -- device code of the HARD-KV Cascade Cache decode step.
//
// Sources: [Abstract] = arXiv abstract on the mlsanity.com page "HARD-KV:
// Head-Adaptive Regularization for Decoding-time KV Compression"; [TS 2.A],
// [TS 2.B], [TS 2.C] = sections "Cascade Cache Hierarchy", "Logits Calibration
// Mechanism", "System-Aware Index Regularization" of the gist.science Technical
// Summary of that paper.
//
// Every kernel runs NTHREADS = 160 threads: warp 4 is a producer that streams
// K/V rows into a 4-slot shared-memory ring with 1-D bulk copies (TMA) and
// mbarriers; warps 0-3 consume one slot each. No tensor cores: a one-query
// decode is a GEMV (about 4 flop per byte), bound by HBM bandwidth.
#pragma once

#include "hkv_device.cuh"

namespace hkv {

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
    int32_t *idx;        // PAD_MAX rows the attention reads (user idx or workspace rows)
    int32_t *idx_user;   // the caller's idx in its own layout (flatten kernel)
    int32_t *offsets;
    float *out, *lse, *m_out, *logZ_out, *P_out;
    char *k_out, *v_out;
    // workspace
    uint32_t *ctl;        // [0] status, [1] ticket, [2] exit count
    uint32_t *score_done; // [units]
    uint32_t *attn_done;  // [units]
    uint32_t *ready;      // [units]
    float *tile_max;      // [units * score_tiles]
    float *part;          // [units * attn_tiles * G * (D + 2)]
    // tiling
    int32_t score_tiles, attn_tiles;  // per unit
    int32_t score_rows;               // rows per score tile
    int32_t attn_toks;                // tokens per attention tile
    int32_t withhold;                 // fault injection: never publish a selection
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

// Compile-time geometry of a (element size, head dim, group size) instance.
template <int ES, int D, int G>
struct Geo {
    static constexpr int ROWB = D * ES;       // bytes of one K or V row
    static constexpr int LPR = ROWB / 16;     // lanes covering one row with 16-byte loads
    static constexpr int RPW = 32 / LPR;      // rows per warp-wide 512-byte load
    static constexpr int VEC = 16 / ES;       // elements in a lane's 16 bytes
    static constexpr int NP = VEC / 2;        // float2 pairs in a lane's 16 bytes
    static constexpr int NB = (LPR / G) < 16 ? (LPR / G) : 16;  // load iterations reduced together
    static constexpr int NV = NB * G;         // partial sums per lane before the reduction
    static constexpr int REP = LPR / NV;      // lanes left holding the same sum afterwards
    static constexpr int SROWS = SLOT_BYTES / ROWB;        // rows per score stage
    static constexpr int SITERS = SLOT_BYTES / 512;        // warp iterations per score stage
    static constexpr int ATOK = (SLOT_BYTES / 2) / ROWB;   // tokens per attention stage
    static constexpr int AITERS = (SLOT_BYTES / 2) / 512;  // warp iterations over the K half
    static constexpr int DPL = D / 32;                     // PV: head-dim elements per lane
    static_assert(G >= 1 && G <= LPR, "group size must not exceed lanes per row");
    static_assert(ATOK * G <= SC_FLOATS, "attention scratch too small");
    static_assert(SITERS % NB == 0 && AITERS % NB == 0 && LPR % NV == 0, "iteration batches");
};

// Shared memory of every kernel. The ring is reused by the select histograms
// and by the attention merge once a tile's stages are consumed.
struct __align__(128) Smem {
    unsigned char ring[NSLOT][SLOT_BYTES];
    float sc[NCW][SC_FLOATS];
    uint64_t full[NSLOT];
    uint64_t empty[NSLOT];
    unsigned long long red[16];
    float redf[16];
    int32_t bc[8];
    unsigned long long bcl[4];
};

struct SelOverlay {  // lives in Smem::ring during a selection
    uint32_t cnt1[HBINS];
    unsigned long long mass1[HBINS];
    uint32_t cnt2[HBINS];
    unsigned long long mass2[HBINS];
};
static_assert(sizeof(SelOverlay) <= sizeof(Smem::ring), "select overlay");

__device__ __forceinline__ void ring_init(Smem &sm)
{
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_fence_init();
    }
    __syncthreads();
}

// The ring's stage sequence: stage q uses slot q % NSLOT for the (q / NSLOT)-th
// time and is consumed by warp q % NCW. Every thread advances `seq` alike.
__device__ __forceinline__ bool producer_acquire(Smem &sm, uint32_t q, const Ctl &c)
{
    const int slot = q % NSLOT;
    const uint32_t use = q / NSLOT;
    return mbar_wait(&sm.empty[slot], (use & 1u) ^ 1u, c);
}

__device__ __forceinline__ bool consumer_acquire(Smem &sm, uint32_t q, const Ctl &c)
{
    const int slot = q % NSLOT;
    const uint32_t use = q / NSLOT;
    return mbar_wait(&sm.full[slot], use & 1u, c);
}

__device__ __forceinline__ void consumer_release(Smem &sm, uint32_t q)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0)
        mbar_arrive(&sm.empty[q % NSLOT]);
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

// Load the lane's slice of the group's G query vectors as float2 pairs.
template <int ES, int D, int G>
__device__ __forceinline__ void load_q(const Params &P, int b, int h, int lane, float2 (&qv)[G][Geo<ES, D, G>::NP])
{
    using Gm = Geo<ES, D, G>;
    const int c = lane % Gm::LPR;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int hq = h * G + g;
        const uint4 w = *reinterpret_cast<const uint4 *>(P.q + ((int64_t)(b * P.Hq + hq) * D + c * Gm::VEC) * ES);
        if constexpr (ES == 2) {
            qv[g][0] = bf16x2_to_float2(w.x);
            qv[g][1] = bf16x2_to_float2(w.y);
            qv[g][2] = bf16x2_to_float2(w.z);
            qv[g][3] = bf16x2_to_float2(w.w);
        } else {
            qv[g][0] = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
            qv[g][1] = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
        }
    }
}

template <int ES>
__device__ __forceinline__ void unpack16(const uint4 &w, float2 (&kv)[16 / ES / 2])
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

// One batch of NB warp iterations over staged rows: per-lane partial dot
// products with the group's queries, reduced across the LPR lanes of a row.
// Returns the lane's reduced value: row (it0 + vi / G) * RPW + lane / LPR, query
// head vi % G, with vi = (lane % LPR) / REP.
template <int ES, int D, int G>
__device__ __forceinline__ float qk_batch(const uint4 *sv, int it0, int lane,
                                          const float2 (&qv)[G][Geo<ES, D, G>::NP])
{
    using Gm = Geo<ES, D, G>;
    float v[Gm::NV];
#pragma unroll
    for (int i = 0; i < Gm::NB; ++i) {
        const uint4 w = sv[(it0 + i) * 32 + lane];
        float2 kv[Gm::NP];
        unpack16<ES>(w, kv);
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

// =============================================================================
// S1 Score tile ([TS 2.B] max-pooled attention logits; [TS 2.A] Tier 2):
// z_j = scale * max_g q_g . k_j for rows [r0, r1) of unit u.
// Returns (in every consumer thread of warp 0 lane 0 ... ) the tile's max via
// Smem::redf after the trailing __syncthreads.
// =============================================================================
template <int ES, int D, int G>
__device__ void score_tile(const Params &P, int u, int r0, int r1, Smem &sm, uint32_t &seq, const Ctl &c,
                           uint64_t policy)
{
    using Gm = Geo<ES, D, G>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = u / P.Hkv, h = u % P.Hkv;
    const int nrows = r1 - r0;
    const int nst = nrows > 0 ? (nrows + Gm::SROWS - 1) / Gm::SROWS : 0;
    const TierP &T = P.sparse;
    const char *kbase = T.k + ((int64_t)b * T.sb + (int64_t)h * T.sh) * ES;

    if (warp == PRODUCER_WARP) {
        const bool contiguous = (T.st == D);
        for (int s = 0; s < nst; ++s) {
            const uint32_t q = seq + s;
            const int slot = q % NSLOT;
            const bool ok = producer_acquire(sm, q, c);
            const int rs = r0 + s * Gm::SROWS;
            const int nr = min(Gm::SROWS, r1 - rs);
            if (lane == 0)
                mbar_arrive_expect_tx(&sm.full[slot], ok ? (uint32_t)(nr * Gm::ROWB) : 0u);
            __syncwarp();
            if (!ok)
                continue;
            if (contiguous) {
                if (lane == 0)
                    bulk_g2s(sm.ring[slot], kbase + (int64_t)rs * T.st * ES, nr * Gm::ROWB, &sm.full[slot], policy);
            } else {
                for (int r = lane; r < nr; r += 32)
                    bulk_g2s(sm.ring[slot] + r * Gm::ROWB, kbase + (int64_t)(rs + r) * T.st * ES, Gm::ROWB,
                             &sm.full[slot], policy);
            }
        }
    } else {
        float2 qv[G][Gm::NP];
        load_q<ES, D, G>(P, b, h, lane, qv);
        float *zu = P.z + (int64_t)u * P.z_stride;
        const int vi = (lane % Gm::LPR) / Gm::REP;
        const bool writer = (lane % Gm::REP) == 0 && (vi % G) == 0;
        float tmax = -INFINITY;
        for (int s = (int)((warp - (int)(seq % NCW) + NCW) % NCW); s < nst; s += NCW) {
            const uint32_t q = seq + s;
            const bool ok = consumer_acquire(sm, q, c);
            const int rs = r0 + s * Gm::SROWS;
            const int nr = min(Gm::SROWS, r1 - rs);
            if (ok) {
                const uint4 *sv = reinterpret_cast<const uint4 *>(sm.ring[q % NSLOT]);
                for (int it0 = 0; it0 < Gm::SITERS && it0 * Gm::RPW < nr; it0 += Gm::NB) {
                    float v = qk_batch<ES, D, G>(sv, it0, lane, qv);
#pragma unroll
                    for (int o = 1; o < G; o <<= 1)
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o * Gm::REP));
                    const int row = (it0 + vi / G) * Gm::RPW + lane / Gm::LPR;
                    if (writer && row < nr) {
                        const float zz = v * P.scale;
                        zu[rs + row] = zz;
                        tmax = fmaxf(tmax, zz);
                    }
                }
            }
            consumer_release(sm, q);
        }
        tmax = warp_max(tmax);
        if (lane == 0)
            sm.redf[warp] = tmax;
    }
    seq += nst;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = sm.redf[0];
        for (int w = 1; w < NCW; ++w)
            t = fmaxf(t, sm.redf[w]);
        sm.redf[NCW] = t;
    }
    __syncthreads();
}

// =============================================================================
// S3 Top-p selection of one unit, whole CTA ([Abstract] Top-p; [TS 2.A]
// head-adaptive budget and hard limits; [TS 2.B] calibrated probabilities).
// Radix descent over the 32-bit order key (11 + 11 + 10 bits) with per-bin
// counts and fixed-point masses.
// =============================================================================
struct Descent {
    uint32_t key;                     // order key of the crossing token
    uint32_t cnt_before;              // tokens with a smaller key (higher score)
    unsigned long long mass_before;   // their fixed-point mass (mass targets only)
    uint32_t cnt_at;                  // tokens with exactly this key
    unsigned long long mass_at;       // their mass (mass targets only)
};

// First bin whose cumulative count (or mass) reaches `target` (1 <= target <=
// total). Result broadcast through sm.bc / sm.bcl.
__device__ __forceinline__ void find_crossing(const uint32_t *cnt, const unsigned long long *mass, int nbins,
                                              bool by_mass, unsigned long long target, Smem &sm)
{
    const int bpt = (nbins + NTHREADS - 1) / NTHREADS;
    const int lo = threadIdx.x * bpt;
    const int hi = min(nbins, lo + bpt);
    unsigned long long my_c = 0, my_m = 0;
    for (int b = lo; b < hi; ++b) {
        my_c += cnt[b];
        if (by_mass)
            my_m += mass[b];
    }
    unsigned long long tot;
    const unsigned long long ex_c = block_exclusive_scan(my_c, sm.red, &tot);
    const unsigned long long ex_m = by_mass ? block_exclusive_scan(my_m, sm.red, &tot) : 0ull;
    const unsigned long long ex = by_mass ? ex_m : ex_c;
    const unsigned long long own = by_mass ? my_m : my_c;
    if (ex < target && target <= ex + own) {
        unsigned long long cc = ex_c, mm = ex_m;
        for (int b = lo; b < hi; ++b) {
            const unsigned long long nc = cc + cnt[b];
            const unsigned long long nm = by_mass ? mm + mass[b] : 0ull;
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
}

__device__ Descent descend(const float *zu, int n, float m, float beta, bool by_mass, unsigned long long target,
                           SelOverlay &ov, Smem &sm)
{
    // level 1: the histogram of all tokens (filled by the caller)
    find_crossing(ov.cnt1, ov.mass1, HBINS, by_mass, target, sm);
    const uint32_t b1 = sm.bc[0];
    unsigned long long cb = sm.bcl[0], mb = sm.bcl[1];
    unsigned long long rem = target - (by_mass ? mb : cb);
    __syncthreads();

    // level 2: next 11 bits among tokens in bin b1
    for (int i = threadIdx.x; i < HBINS; i += NTHREADS) {
        ov.cnt2[i] = 0;
        ov.mass2[i] = 0;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += NTHREADS) {
        const float zj = __ldcg(zu + j);
        const uint32_t key = score_key(zj);
        if ((key >> (L2_BITS + L3_BITS)) != b1)
            continue;
        const uint32_t bin = (key >> L3_BITS) & ((1u << L2_BITS) - 1);
        atomicAdd(&ov.cnt2[bin], 1u);
        if (by_mass)
            atomicAdd(&ov.mass2[bin], wfix(zj, m, beta));
    }
    __syncthreads();
    find_crossing(ov.cnt2, ov.mass2, 1 << L2_BITS, by_mass, rem, sm);
    const uint32_t b2 = sm.bc[0];
    cb += sm.bcl[0];
    mb += sm.bcl[1];
    rem -= by_mass ? sm.bcl[1] : sm.bcl[0];
    __syncthreads();

    // level 3: last 10 bits among tokens with the 22-bit prefix
    const uint32_t prefix = (b1 << L2_BITS) | b2;
    for (int i = threadIdx.x; i < (1 << L3_BITS); i += NTHREADS) {
        ov.cnt2[i] = 0;
        ov.mass2[i] = 0;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += NTHREADS) {
        const float zj = __ldcg(zu + j);
        const uint32_t key = score_key(zj);
        if ((key >> L3_BITS) != prefix)
            continue;
        const uint32_t bin = key & ((1u << L3_BITS) - 1);
        atomicAdd(&ov.cnt2[bin], 1u);
        if (by_mass)
            atomicAdd(&ov.mass2[bin], wfix(zj, m, beta));
    }
    __syncthreads();
    find_crossing(ov.cnt2, ov.mass2, 1 << L3_BITS, by_mass, rem, sm);
    const uint32_t b3 = sm.bc[0];
    Descent d;
    d.key = (prefix << L3_BITS) | b3;
    d.cnt_before = (uint32_t)(cb + sm.bcl[0]);
    d.mass_before = mb + sm.bcl[1];
    d.cnt_at = ov.cnt2[b3];
    d.mass_at = ov.mass2[b3];
    __syncthreads();
    return d;
}

struct Selection {
    int32_t k, kstar;
    hkv_cut cut;
    uint32_t key;                 // order key of the cut (0 when k = 0)
    unsigned long long Z;         // fixed-point normaliser
};

// Budget and cut of one unit; every thread of the CTA calls it and gets the
// same result. `m` is the unit's maximum score.
__device__ Selection select_unit(const float *zu, int n, float m, float beta, float p, int bmin, int bmax,
                                 Smem &sm)
{
    SelOverlay &ov = *reinterpret_cast<SelOverlay *>(sm.ring);
    Selection r{};
    for (int i = threadIdx.x; i < HBINS; i += NTHREADS) {
        ov.cnt1[i] = 0;
        ov.mass1[i] = 0;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += NTHREADS) {
        const float zj = __ldcg(zu + j);
        const uint32_t bin = score_key(zj) >> (L2_BITS + L3_BITS);
        atomicAdd(&ov.cnt1[bin], 1u);
        atomicAdd(&ov.mass1[bin], wfix(zj, m, beta));
    }
    __syncthreads();
    unsigned long long part = 0;
    for (int i = threadIdx.x; i < HBINS; i += NTHREADS)
        part += ov.mass1[i];
    r.Z = block_sum_u64(part, sm.red);

    int kstar;
    bool have_mass_cut = false;
    Descent dm{};
    unsigned long long T = 0;
    if (n == 0)
        kstar = 0;
    else if (p >= 1.0f)
        kstar = n;
    else if (p <= 0.0f)
        kstar = 0;
    else {
        double t = ceil((double)p * (double)r.Z);
        T = t < 1.0 ? 1ull : (unsigned long long)t;
        if (T > r.Z)
            T = r.Z;
        dm = descend(zu, n, m, beta, true, T, ov, sm);
        const unsigned long long w_at = dm.mass_at / dm.cnt_at;
        const unsigned long long need = T - dm.mass_before;
        const unsigned long long ties = (need + w_at - 1) / w_at;
        kstar = (int)(dm.cnt_before + ties);
        have_mass_cut = true;
    }
    int k = min(kstar, bmax);
    k = max(k, bmin);
    k = min(k, n);
    r.k = k;
    r.kstar = kstar;
    if (k == 0) {
        r.key = 0;
        r.cut = hkv_cut{0.0f, 0, 0, kstar};
    } else if (have_mass_cut && k == kstar) {
        r.key = dm.key;
        r.cut = hkv_cut{key_score(dm.key), (int32_t)dm.cnt_before, (int32_t)(k - dm.cnt_before), kstar};
    } else {
        const Descent dc = descend(zu, n, m, beta, false, (unsigned long long)k, ov, sm);
        r.key = dc.key;
        r.cut = hkv_cut{key_score(dc.key), (int32_t)dc.cnt_before, (int32_t)(k - dc.cnt_before), kstar};
    }
    __syncthreads();
    return r;
}

// =============================================================================
// S4 Index Regularization of one unit, whole CTA ([TS 2.C] Flatten Index):
// order-preserving compaction of {key < cut key} + the first n_tie tokens with
// key == cut key into row[0, k); PAD_MAX rows are padded with -1 to `pad`.
// =============================================================================
__device__ void compact_unit(const float *zu, int n, uint32_t cut_key, int n_tie, int k, int32_t *row, int pad,
                             unsigned long long *red)
{
    constexpr int E = 8;
    unsigned long long lt_carry = 0, eq_carry = 0;
    if (k > 0) {
        for (int base = 0; base < n; base += NTHREADS * E) {
            const int j0 = base + threadIdx.x * E;
            uint32_t keys[E];
            uint32_t nlt = 0, neq = 0;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = j0 + e;
                keys[e] = j < n ? score_key(__ldcg(zu + j)) : 0xffffffffu;
                const bool valid = j < n;
                nlt += (valid && keys[e] < cut_key) ? 1u : 0u;
                neq += (valid && keys[e] == cut_key) ? 1u : 0u;
            }
            unsigned long long tot;
            const unsigned long long ex = block_exclusive_scan(((unsigned long long)neq << 32) | nlt, red, &tot);
            const unsigned long long eq_before = eq_carry + (ex >> 32);
            const unsigned long long lt_before = lt_carry + (ex & 0xffffffffull);
            unsigned long long pos = lt_before + min(eq_before, (unsigned long long)n_tie);
            unsigned long long eq_rank = eq_before;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = j0 + e;
                if (j >= n)
                    break;
                bool take = keys[e] < cut_key;
                if (keys[e] == cut_key) {
                    take = eq_rank < (unsigned long long)n_tie;
                    ++eq_rank;
                }
                if (take && pos < (unsigned long long)k)  // a caller's inconsistent cut stays in the row
                    row[pos++] = j;
            }
            lt_carry += tot & 0xffffffffull;
            eq_carry += tot >> 32;
        }
    }
    for (int i = k + threadIdx.x; i < pad; i += NTHREADS)
        row[i] = -1;
}

// =============================================================================
// S5 attention tile ([TS 2.A] the three tiers; [TS 2.C] Sparse Loading):
// tokens [t0, t1) of dense[0, W) ++ sparse[idx[0, k)] ++ condensed[0, Cn) for
// the G query heads of unit u. Writes the tile's unnormalised partial
// (o[G][D], m[G], l[G]) to `part`.
// =============================================================================
template <int ES, int D, int G>
__device__ void attn_tile(const Params &P, int u, int t0, int t1, const int32_t *idx_row, int W, int k, int Cn,
                          int n_sparse, float *part, Smem &sm, uint32_t &seq, const Ctl &c, uint64_t policy)
{
    using Gm = Geo<ES, D, G>;
    constexpr int NPV = Gm::DPL / 2;  // float2 pairs of the lane's head-dim slice
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = u / P.Hkv, h = u % P.Hkv;
    const int ntok = t1 - t0;
    const int nst = ntok > 0 ? (ntok + Gm::ATOK - 1) / Gm::ATOK : 0;

    float m_run[G], l_run[G];
    float2 o[G][NPV];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m_run[g] = -INFINITY;
        l_run[g] = 0.f;
#pragma unroll
        for (int e = 0; e < NPV; ++e)
            o[g][e] = make_float2(0.f, 0.f);
    }

    if (warp == PRODUCER_WARP) {
        for (int s = 0; s < nst; ++s) {
            const uint32_t q = seq + s;
            const int slot = q % NSLOT;
            const bool ok = producer_acquire(sm, q, c);
            const int ts = t0 + s * Gm::ATOK;
            const int nt = min(Gm::ATOK, t1 - ts);
            if (lane == 0)
                mbar_arrive_expect_tx(&sm.full[slot], ok ? (uint32_t)(2 * nt * Gm::ROWB) : 0u);
            __syncwarp();
            if (!ok)
                continue;
            for (int i = lane; i < nt; i += 32) {
                const int t = ts + i;
                const char *kb, *vb;
                int64_t off;
                if (t < W) {
                    kb = P.dense.k;
                    vb = P.dense.v;
                    off = (int64_t)b * P.dense.sb + (int64_t)h * P.dense.sh + (int64_t)t * P.dense.st;
                } else if (t < W + k) {
                    int j = __ldcg(idx_row + (t - W));
                    if (j < 0 || j >= n_sparse) {
                        raise_flag(c, HKV_DEV_BAD_INDEX);
                        j = 0;
                    }
                    kb = P.sparse.k;
                    vb = P.sparse.v;
                    off = (int64_t)b * P.sparse.sb + (int64_t)h * P.sparse.sh + (int64_t)j * P.sparse.st;
                } else {
                    kb = P.cond.k;
                    vb = P.cond.v;
                    off = (int64_t)b * P.cond.sb + (int64_t)h * P.cond.sh + (int64_t)(t - W - k) * P.cond.st;
                }
                bulk_g2s(sm.ring[slot] + i * Gm::ROWB, kb + off * ES, Gm::ROWB, &sm.full[slot], policy);
                bulk_g2s(sm.ring[slot] + SLOT_BYTES / 2 + i * Gm::ROWB, vb + off * ES, Gm::ROWB, &sm.full[slot],
                         policy);
            }
        }
    } else {
        float2 qv[G][Gm::NP];
        load_q<ES, D, G>(P, b, h, lane, qv);
        const float scale = P.scale;
        const int vi = (lane % Gm::LPR) / Gm::REP;
        const bool writer = (lane % Gm::REP) == 0;
        float *sc = sm.sc[warp];
        for (int s = (int)((warp - (int)(seq % NCW) + NCW) % NCW); s < nst; s += NCW) {
            const uint32_t q = seq + s;
            const bool ok = consumer_acquire(sm, q, c);
            const int nt = min(Gm::ATOK, t1 - (t0 + s * Gm::ATOK));
            if (ok) {
                const unsigned char *slotp = sm.ring[q % NSLOT];
                const uint4 *kv4 = reinterpret_cast<const uint4 *>(slotp);
                // logits of the stage's tokens for all G query heads
                for (int it0 = 0; it0 < Gm::AITERS && it0 * Gm::RPW < nt; it0 += Gm::NB) {
                    const float v = qk_batch<ES, D, G>(kv4, it0, lane, qv);
                    const int row = (it0 + vi / G) * Gm::RPW + lane / Gm::LPR;
                    if (writer && row < nt)
                        sc[row * G + (vi % G)] = v * scale;
                }
                __syncwarp();
                // online softmax: lane owns rows lane, lane + 32 of the stage
                float alpha[G];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float mx = -INFINITY;
                    for (int r = lane; r < nt; r += 32)
                        mx = fmaxf(mx, sc[r * G + g]);
                    mx = warp_max(mx);
                    const float m_new = fmaxf(m_run[g], mx);
                    alpha[g] = (m_new == -INFINITY) ? 1.0f : expf(m_run[g] - m_new);
                    float lp = 0.f;
                    for (int r = lane; r < nt; r += 32) {
                        const float pr = (m_new == -INFINITY) ? 0.0f : expf(sc[r * G + g] - m_new);
                        sc[r * G + g] = pr;
                        lp += pr;
                    }
                    l_run[g] = l_run[g] * alpha[g] + lp;
                    m_run[g] = m_new;
                }
                __syncwarp();
                // o = alpha o + sum_t p_t v_t over the lane's head-dim slice
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int e = 0; e < NPV; ++e) {
                        o[g][e].x *= alpha[g];
                        o[g][e].y *= alpha[g];
                    }
                const unsigned char *vbase = slotp + SLOT_BYTES / 2 + lane * Gm::DPL * ES;
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
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float pr = sc[r * G + g];
                        const float2 pp = make_float2(pr, pr);
#pragma unroll
                        for (int e = 0; e < NPV; ++e)
                            o[g][e] = ffma2(pp, vv[e], o[g][e]);
                    }
                }
                __syncwarp();
            }
            consumer_release(sm, q);
        }
#pragma unroll
        for (int g = 0; g < G; ++g)
            l_run[g] = warp_sum(l_run[g]);
    }
    seq += nst;
    // Every stage of the tile has been consumed, so all its copies have landed
    // and the ring is free for the warps' states.
    __syncthreads();
    float *mw = reinterpret_cast<float *>(sm.ring[0]);  // [NCW][G]
    float *lw = mw + NCW * G;                           // [NCW][G]
    float *ow = lw + NCW * G;                           // [NCW][G][D]
    if (warp < NCW) {
        if (lane == 0)
#pragma unroll
            for (int g = 0; g < G; ++g) {
                mw[warp * G + g] = m_run[g];
                lw[warp * G + g] = l_run[g];
            }
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < NPV; ++e) {
                ow[(warp * G + g) * D + lane * Gm::DPL + 2 * e] = o[g][e].x;
                ow[(warp * G + g) * D + lane * Gm::DPL + 2 * e + 1] = o[g][e].y;
            }
    }
    __syncthreads();
    // tile partial: part[g*(D+2) + d] = o (unnormalised), [D] = m, [D+1] = l
    for (int i = threadIdx.x; i < G * (D + 2); i += NTHREADS) {
        const int g = i / (D + 2), d = i % (D + 2);
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NCW; ++w)
            M = fmaxf(M, mw[w * G + g]);
        float acc = 0.f;
        if (d == D) {
            acc = M;
        } else {
#pragma unroll
            for (int w = 0; w < NCW; ++w) {
                const float mwg = mw[w * G + g];
                if (mwg == -INFINITY)
                    continue;
                const float f = expf(mwg - M);
                acc += (d < D ? ow[(w * G + g) * D + d] : lw[w * G + g]) * f;
            }
        }
        part[i] = acc;
    }
    __syncthreads();
}

// Merge the unit's attention tile partials (fixed order) into out and lse.
template <int D, int G>
__device__ void merge_unit(const Params &P, int u, const float *parts, int ntiles)
{
    const int b = u / P.Hkv, h = u % P.Hkv;
    for (int i = threadIdx.x; i < G * D; i += NTHREADS) {
        const int g = i / D, d = i % D;
        float M = -INFINITY;
        for (int t = 0; t < ntiles; ++t)
            M = fmaxf(M, __ldcg(parts + (int64_t)t * G * (D + 2) + g * (D + 2) + D));
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
            for (int t = 0; t < ntiles; ++t) {
                const float *pt = parts + (int64_t)t * G * (D + 2) + g * (D + 2);
                const float mt = __ldcg(pt + D);
                if (mt == -INFINITY)
                    continue;
                const float f = expf(mt - M);
                L += __ldcg(pt + D + 1) * f;
                O += __ldcg(pt + d) * f;
            }
        }
        const int hq = h * G + g;
        P.out[((int64_t)b * P.Hq + hq) * D + d] = (M == -INFINITY) ? 0.0f : O / L;
        if (d == 0 && P.lse != nullptr)
            P.lse[(int64_t)b * P.Hq + hq] = (M == -INFINITY) ? -INFINITY : M + logf(L);
    }
}

}  // namespace hkv
