// hkv_api.cu -- kernels and C ABI of the HARD-KV Cascade Cache decode step.
//
// Sources: [Abstract] = arXiv abstract on the mlsanity.com page "HARD-KV:
// Head-Adaptive Regularization for Decoding-time KV Compression"; [TS 2.A],
// [TS 2.B], [TS 2.C] = sections of the gist.science Technical Summary of that
// paper ("Cascade Cache Hierarchy", "Logits Calibration Mechanism",
// "System-Aware Index Regularization").
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "hkv_kernels.cuh"

namespace hkv {

// Work per tile: 256 KiB of sparse keys per score tile, 64 KiB of keys (and as
// much of values) per attention tile.
constexpr int SCORE_TILE_BYTES = 256 * 1024;
constexpr int ATTN_TILE_BYTES = 64 * 1024;

// =============================================================================
// Kernels
// =============================================================================

// S1 standalone: one score tile per CTA.
template <int ES, int D, int G>
__global__ void __launch_bounds__(NTHREADS) k_score(const __grid_constant__ Params P)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const Ctl c = make_ctl(P);
    const int u = blockIdx.x / P.score_tiles, t = blockIdx.x % P.score_tiles;
    const int n = tier_len(P.sparse, u, c);
    const int r0 = t * P.score_rows, r1 = min(n, r0 + P.score_rows);
    if (r0 >= r1)
        return;
    ring_init(sm);
    uint32_t seq = 0;
    score_tile<ES, D, G>(P, u, r0, r1, sm, seq, c, evict_first_policy());
}

// S2 standalone: one unit per CTA.
__global__ void __launch_bounds__(NTHREADS) k_calibrate(const __grid_constant__ Params P)
{
    __shared__ unsigned long long red[16];
    __shared__ float redf[16];
    const Ctl c = make_ctl(P);
    const int u = blockIdx.x;
    const int n = tier_len(P.sparse, u, c);
    const float *zu = P.z + (int64_t)u * P.z_stride;
    float mx = -INFINITY;
    for (int j = threadIdx.x; j < n; j += NTHREADS)
        mx = fmaxf(mx, __ldcg(zu + j));
    const float m = block_max(mx, redf);
    const float beta = unit_beta(P, u, c);
    unsigned long long part = 0;
    for (int j = threadIdx.x; j < n; j += NTHREADS)
        part += wfix(__ldcg(zu + j), m, beta);
    const unsigned long long Z = block_sum_u64(part, red);
    if (P.P_out != nullptr && n > 0) {
        const float inv = (float)(1099511627776.0 / (double)Z);
        float *Pu = P.P_out + (int64_t)u * P.z_stride;
        for (int j = threadIdx.x; j < n; j += NTHREADS) {
            const float zj = __ldcg(zu + j);
            const float w = (zj == m || beta == 0.0f) ? 1.0f : expf(beta * (zj - m));
            Pu[j] = w * inv;
        }
    }
    if (threadIdx.x == 0) {
        P.m_out[u] = m;
        P.logZ_out[u] = n > 0 ? (float)(log((double)Z) - WFIX_BITS * 0.6931471805599453) : -INFINITY;
    }
}

// S3 standalone: one unit per CTA.
__global__ void __launch_bounds__(NTHREADS) k_select(const __grid_constant__ Params P)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const Ctl c = make_ctl(P);
    const int u = blockIdx.x;
    const int n = tier_len(P.sparse, u, c);
    const float *zu = P.z + (int64_t)u * P.z_stride;
    float mx = -INFINITY;
    for (int j = threadIdx.x; j < n; j += NTHREADS)
        mx = fmaxf(mx, __ldcg(zu + j));
    const float m = block_max(mx, sm.redf);
    const Selection s = select_unit(zu, n, m, unit_beta(P, u, c), unit_p(P, u, c), P.bmin, P.bmax, sm);
    if (threadIdx.x == 0) {
        P.sel_len[u] = s.k;
        P.cut[u] = s.cut;
    }
}

// Rewrite Cache ([TS 2.C]): copy the k selected K/V rows of unit u, listed in
// `row`, to rows dst_row0 .. dst_row0 + k - 1 of k_out / v_out.
__device__ void rewrite_rows(const Params &P, int u, const int32_t *row, int k, int64_t dst_row0, int es,
                             const Ctl &c, int n_sparse)
{
    const int b = u / P.Hkv, h = u % P.Hkv;
    const int vec_per_row = P.D * es / 16;
    const int64_t total = (int64_t)k * vec_per_row;
    for (int64_t i = threadIdx.x; i < total; i += NTHREADS) {
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

// Exclusive scan position of unit u in the FLAT_SUM layout.
__device__ int64_t flat_offset(const Params &P, int u, unsigned long long *red)
{
    unsigned long long part = 0;
    for (int i = threadIdx.x; i < u; i += NTHREADS)
        part += (unsigned long long)max(0, __ldcg(P.sel_len + i));
    return (int64_t)block_sum_u64(part, red);
}

// S4 standalone ([TS 2.C]): compaction of one unit per CTA from its cut, into
// the caller's layout, plus the optional Rewrite Cache copy.
template <int ES>
__global__ void __launch_bounds__(NTHREADS) k_compact(const __grid_constant__ Params P)
{
    __shared__ unsigned long long red[16];
    const Ctl c = make_ctl(P);
    const int u = blockIdx.x;
    const int n = tier_len(P.sparse, u, c);
    const float *zu = P.z + (int64_t)u * P.z_stride;
    int k = __ldcg(P.sel_len + u);
    const hkv_cut ct = P.cut[u];
    if (k < 0 || k > n || k > P.bmax || ct.n_above < 0 || ct.n_tie < 0 || ct.n_above + ct.n_tie != k) {
        raise_flag(c, HKV_DEV_BAD_INDEX);
        k = 0;
    }
    int64_t off;
    if (P.layout == HKV_LAYOUT_FLAT_SUM) {
        off = flat_offset(P, u, red);
        if (threadIdx.x == 0) {
            P.offsets[u] = (int32_t)off;
            if (u == P.units - 1)
                P.offsets[P.units] = (int32_t)(off + max(0, __ldcg(P.sel_len + u)));
        }
    } else {
        off = (int64_t)u * P.bmax;
    }
    int32_t *row = P.idx + off;
    compact_unit(zu, n, k > 0 ? score_key(ct.z_cut) : 0u, ct.n_tie, k, row,
                 P.layout == HKV_LAYOUT_PAD_MAX ? P.bmax : k, red);
    if (P.k_out != nullptr) {
        __syncthreads();
        rewrite_rows(P, u, row, k, off, ES, c, n);
    }
}

// S5 standalone: one attention tile per CTA; the last tile of a unit merges it.
template <int ES, int D, int G>
__global__ void __launch_bounds__(NTHREADS) k_decode(const __grid_constant__ Params P)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const Ctl c = make_ctl(P);
    const int u = blockIdx.x / P.attn_tiles, s = blockIdx.x % P.attn_tiles;
    const int W = tier_len(P.dense, u, c), Cn = tier_len(P.cond, u, c);
    const int n = tier_len(P.sparse, u, c);
    int k = P.sparse.len ? __ldcg(P.sel_len + u) : 0;
    if (k < 0 || k > n || k > P.bmax) {
        raise_flag(c, HKV_DEV_BAD_INDEX);
        k = max(0, min(k, min(n, P.bmax)));
    }
    const int32_t *idx_row =
        P.layout == HKV_LAYOUT_FLAT_SUM ? P.idx + __ldcg(P.offsets + u) : P.idx + (int64_t)u * P.bmax;
    const int total = W + k + Cn;
    const int t0 = s * P.attn_toks, t1 = min(total, t0 + P.attn_toks);
    float *parts = P.part + (int64_t)u * P.attn_tiles * G * (D + 2);
    ring_init(sm);
    if (t0 < t1) {
        uint32_t seq = 0;
        attn_tile<ES, D, G>(P, u, t0, t1, idx_row, W, k, Cn, n, parts + (int64_t)s * G * (D + 2), sm, seq, c,
                            evict_first_policy());
    }
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t prev = atomicAdd(P.attn_done + u, 1u);
        sm.bc[0] = (prev == (uint32_t)P.attn_tiles - 1) ? 1 : 0;
    }
    __syncthreads();
    if (sm.bc[0]) {
        __threadfence();
        merge_unit<D, G>(P, u, parts, (total + P.attn_toks - 1) / P.attn_toks);
        if (threadIdx.x == 0)
            P.attn_done[u] = 0;
    }
}

// FLAT_SUM rows and Rewrite Cache copies after the fused step: one unit per CTA.
template <int ES>
__global__ void __launch_bounds__(NTHREADS) k_flatten(const __grid_constant__ Params P)
{
    const Ctl c = make_ctl(P);
    const int u = blockIdx.x;
    const int n = tier_len(P.sparse, u, c);
    const int k = max(0, min(__ldcg(P.sel_len + u), min(n, P.bmax)));
    const int32_t *src = P.idx + (int64_t)u * P.bmax;
    int64_t off = (int64_t)u * P.bmax;
    if (P.layout == HKV_LAYOUT_FLAT_SUM) {
        __shared__ unsigned long long red[16];
        off = flat_offset(P, u, red);
        for (int i = threadIdx.x; i < k; i += NTHREADS)
            P.idx_user[off + i] = __ldcg(src + i);
        if (threadIdx.x == 0) {
            P.offsets[u] = (int32_t)off;
            if (u == P.units - 1)
                P.offsets[P.units] = (int32_t)(off + k);
        }
    }
    if (P.k_out != nullptr)
        rewrite_rows(P, u, src, k, off, ES, c, n);
}

// S1..S5 fused: persistent CTAs take tickets in order -- every score tile
// first (unit-major), then every attention tile. The CTA finishing a unit's
// last score tile selects and compacts that unit and publishes it; attention
// tiles of the unit wait (bounded) for that. A unit's last attention tile
// merges the unit. Tickets only wait on tickets issued before them, whose
// CTAs are running, so the schedule cannot deadlock.
template <int ES, int D, int G>
__global__ void __launch_bounds__(NTHREADS) k_step(const __grid_constant__ Params P)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const Ctl c = make_ctl(P);
    const uint64_t policy = evict_first_policy();
    const int n_score = P.units * P.score_tiles;
    const int n_total = n_score + P.units * P.attn_tiles;
    ring_init(sm);
    uint32_t seq = 0;
    for (;;) {
        if (threadIdx.x == 0)
            sm.bc[1] = (int32_t)atomicAdd(P.ctl + 1, 1u);
        __syncthreads();
        const int t = sm.bc[1];
        __syncthreads();
        if (t >= n_total)
            break;
        if (t < n_score) {
            const int u = t / P.score_tiles, ct = t % P.score_tiles;
            const int n = tier_len(P.sparse, u, c);
            const int r0 = ct * P.score_rows, r1 = min(n, r0 + P.score_rows);
            float tmax = -INFINITY;
            if (r0 < r1) {
                score_tile<ES, D, G>(P, u, r0, r1, sm, seq, c, policy);
                tmax = sm.redf[NCW];
            }
            if (threadIdx.x == 0) {
                P.tile_max[(int64_t)u * P.score_tiles + ct] = tmax;
                __threadfence();
                const uint32_t prev = atomicAdd(P.score_done + u, 1u);
                sm.bc[2] = (prev == (uint32_t)P.score_tiles - 1) ? 1 : 0;
            }
            __syncthreads();
            if (!sm.bc[2])
                continue;
            // Last score tile of unit u: Logits Calibration, Top-p, compaction.
            __threadfence();
            if (threadIdx.x == 0) {
                float m = -INFINITY;
                for (int i = 0; i < P.score_tiles; ++i)
                    m = fmaxf(m, __ldcg(P.tile_max + (int64_t)u * P.score_tiles + i));
                sm.redf[8] = m;
            }
            __syncthreads();
            const float m = sm.redf[8];
            const float *zu = P.z + (int64_t)u * P.z_stride;
            const Selection s = select_unit(zu, n, m, unit_beta(P, u, c), unit_p(P, u, c), P.bmin, P.bmax, sm);
            compact_unit(zu, n, s.key, s.cut.n_tie, s.k, P.idx + (int64_t)u * P.bmax, P.bmax, sm.red);
            if (threadIdx.x == 0) {
                P.sel_len[u] = s.k;
                if (P.cut)
                    P.cut[u] = s.cut;
                if (P.m_out)
                    P.m_out[u] = m;
                if (P.logZ_out)
                    P.logZ_out[u] = n > 0 ? (float)(log((double)s.Z) - WFIX_BITS * 0.6931471805599453) : -INFINITY;
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                __threadfence();
                P.score_done[u] = 0;
                if (!P.withhold)
                    st_release(P.ready + u, 1u);
            }
        } else {
            const int a = t - n_score;
            const int u = a / P.attn_tiles, st = a % P.attn_tiles;
            if (threadIdx.x == 0) {
                bool ok = ld_acquire(P.ready + u) != 0;
                if (!ok) {
                    const uint64_t t0 = global_ns();
                    while (!ok) {
                        __nanosleep(200);
                        ok = ld_acquire(P.ready + u) != 0;
                        if (ok || timed_out(c))
                            break;
                        if (global_ns() - t0 > c.wait_ns) {
                            raise_flag(c, HKV_DEV_TIMEOUT);
                            break;
                        }
                    }
                }
                sm.bc[3] = ok ? 1 : 0;
            }
            __syncthreads();
            const bool ready = sm.bc[3] != 0;
            const int W = tier_len(P.dense, u, c), Cn = tier_len(P.cond, u, c);
            const int n = tier_len(P.sparse, u, c);
            const int k = ready ? max(0, min(__ldcg(P.sel_len + u), min(n, P.bmax))) : 0;
            const int total = W + k + Cn;
            const int t0 = st * P.attn_toks, t1 = min(total, t0 + P.attn_toks);
            float *parts = P.part + (int64_t)u * P.attn_tiles * G * (D + 2);
            if (t0 < t1)
                attn_tile<ES, D, G>(P, u, t0, t1, P.idx + (int64_t)u * P.bmax, W, k, Cn, n,
                                    parts + (int64_t)st * G * (D + 2), sm, seq, c, policy);
            if (threadIdx.x == 0) {
                __threadfence();
                const uint32_t prev = atomicAdd(P.attn_done + u, 1u);
                sm.bc[4] = (prev == (uint32_t)P.attn_tiles - 1) ? 1 : 0;
            }
            __syncthreads();
            if (sm.bc[4]) {
                __threadfence();
                merge_unit<D, G>(P, u, parts, (total + P.attn_toks - 1) / P.attn_toks);
                __syncthreads();
                if (threadIdx.x == 0) {
                    P.attn_done[u] = 0;
                    P.ready[u] = 0;
                }
            }
        }
    }
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t prev = atomicAdd(P.ctl + 2, 1u);
        if (prev == gridDim.x - 1) {
            P.ctl[1] = 0;
            P.ctl[2] = 0;
        }
    }
}

// =============================================================================
// Host side
// =============================================================================

std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_wait_ns{1000000000ull};
std::atomic<int32_t> g_withhold{0};

struct WsLayout {
    size_t ctl, score_done, attn_done, ready, tile_max, zbuf, idxbuf, part, cutbuf, total;
    int64_t z_stride;
    int score_tiles, attn_tiles, score_rows, attn_toks;
};

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static int es_of(hkv_dtype d) { return d == HKV_BF16 ? 2 : 4; }

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

static WsLayout layout_of(const hkv_problem *p, const hkv_tier *dense, const hkv_tier *sparse,
                          const hkv_tier *cond)
{
    WsLayout L{};
    const int es = es_of(p->dtype);
    const int64_t units = (int64_t)p->B * p->Hkv;
    const int G = p->Hq / p->Hkv;
    const int ncap = sparse ? sparse->cap : 0;
    const int wcap = dense ? dense->cap : 0;
    const int ccap = cond ? cond->cap : 0;
    L.score_rows = SCORE_TILE_BYTES / (p->D * es);
    L.attn_toks = ATTN_TILE_BYTES / (p->D * es);
    L.score_tiles = std::max(1, (ncap + L.score_rows - 1) / L.score_rows);
    const int64_t max_tokens = (int64_t)wcap + std::min<int64_t>(p->bmax, ncap) + ccap;
    L.attn_tiles = (int)std::max<int64_t>(1, (max_tokens + L.attn_toks - 1) / L.attn_toks);
    L.z_stride = (int64_t)align_up((size_t)std::max(ncap, 1), 4);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes, 256);
        return at;
    };
    L.ctl = take(256);
    L.score_done = take(units * 4);
    L.attn_done = take(units * 4);
    L.ready = take(units * 4);
    L.tile_max = take(units * L.score_tiles * 4);
    L.cutbuf = take(units * sizeof(hkv_cut));
    L.idxbuf = take(units * (size_t)std::max(p->bmax, 1) * 4);
    L.part = take((size_t)units * L.attn_tiles * G * (p->D + 2) * 4);
    L.zbuf = take((size_t)units * L.z_stride * 4);
    L.total = o;
    return L;
}

static Params base_params(const hkv_problem *p, const WsLayout &L, char *ws)
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
    P.score_tiles = L.score_tiles;
    P.attn_tiles = L.attn_tiles;
    P.score_rows = L.score_rows;
    P.attn_toks = L.attn_toks;
    P.z_stride = L.z_stride;
    P.wait_ns = g_wait_ns.load();
    P.withhold = g_withhold.load();
    if (ws) {
        P.ctl = reinterpret_cast<uint32_t *>(ws + L.ctl);
        P.score_done = reinterpret_cast<uint32_t *>(ws + L.score_done);
        P.attn_done = reinterpret_cast<uint32_t *>(ws + L.attn_done);
        P.ready = reinterpret_cast<uint32_t *>(ws + L.ready);
        P.tile_max = reinterpret_cast<float *>(ws + L.tile_max);
        P.part = reinterpret_cast<float *>(ws + L.part);
    }
    return P;
}

static hkv_status check_ws(void *ws, size_t ws_bytes, const WsLayout &L)
{
    if (ws == nullptr || ((uintptr_t)ws & 255) || ws_bytes < L.total)
        return HKV_ERR_WORKSPACE;
    return HKV_OK;
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

// Per-device cache of kernel attributes (dynamic smem opt-in, occupancy).
struct KernelInfo {
    const void *fn;
    int device;
    int blocks_per_sm;
};
static std::mutex g_mu;
static KernelInfo g_info[256];
static int g_ninfo = 0;

static hkv_status prepare(const void *fn, size_t smem, int *blocks_per_sm)
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
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, fn, NTHREADS, smem) != cudaSuccess)
        return HKV_ERR_CUDA;
    if (g_ninfo < 256)
        g_info[g_ninfo++] = KernelInfo{fn, dev, bps};
    if (blocks_per_sm)
        *blocks_per_sm = bps;
    return HKV_OK;
}

template <typename K>
static hkv_status launch(K kernel, int grid, size_t smem, cudaStream_t stream, const Params &P)
{
    if (grid <= 0)
        return HKV_OK;
    hkv_status s = prepare((const void *)kernel, smem, nullptr);
    if (s != HKV_OK)
        return s;
    kernel<<<grid, NTHREADS, smem, stream>>>(P);
    g_launches.fetch_add(1);
    return cudaGetLastError() == cudaSuccess ? HKV_OK : HKV_ERR_CUDA;
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
    static hkv_status run(const Params &P, int grid, cudaStream_t s)
    {
        return launch(k_score<ES, D, G>, grid, sizeof(Smem), s, P);
    }
};

template <int ES, int D, int G>
struct RunDecode {
    static hkv_status run(const Params &P, int grid, cudaStream_t s)
    {
        return launch(k_decode<ES, D, G>, grid, sizeof(Smem), s, P);
    }
};

template <int ES, int D, int G>
struct RunStep {
    static hkv_status run(const Params &P, int max_grid, cudaStream_t s)
    {
        int bps = 0;
        hkv_status st = prepare((const void *)k_step<ES, D, G>, sizeof(Smem), &bps);
        if (st != HKV_OK)
            return st;
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return HKV_ERR_CUDA;
        const int grid = std::min(max_grid, std::max(1, bps) * sms);
        return launch(k_step<ES, D, G>, grid, sizeof(Smem), s, P);
    }
};

}  // namespace hkv

using namespace hkv;

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

}  // extern "C"

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
    *P = base_params(prob, *L, static_cast<char *>(ws));
    P->dense = tier_p(dense);
    P->sparse = tier_p(sparse);
    P->cond = tier_p(cond);
    return HKV_OK;
}

bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

}  // namespace

extern "C" {

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
    return dispatch<RunScore>(prob, P, P.units * P.score_tiles, (cudaStream_t)stream);
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
    return launch(k_calibrate, P.units, 0, (cudaStream_t)stream, P);
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
    return launch(k_select, P.units, sizeof(Smem), (cudaStream_t)stream, P);
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
    if (prob->dtype == HKV_BF16)
        return launch(k_compact<2>, P.units, 0, (cudaStream_t)stream, P);
    return launch(k_compact<4>, P.units, 0, (cudaStream_t)stream, P);
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
    P.q = static_cast<const char *>(q);
    P.idx = const_cast<int32_t *>(idx);
    P.offsets = const_cast<int32_t *>(offsets);
    P.sel_len = const_cast<int32_t *>(sel_len);
    P.out = out;
    P.lse = lse;
    return dispatch<RunDecode>(prob, P, P.units * P.attn_tiles, (cudaStream_t)stream);
}

hkv_status hkv_step(const hkv_problem *prob, const void *q, const hkv_tier *dense, const hkv_tier *sparse,
                    const hkv_tier *condensed, const hkv_step_out *o, void *ws, size_t ws_bytes,
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
    if (P.units == 0)
        return HKV_OK;
    char *wsb = static_cast<char *>(ws);
    P.q = static_cast<const char *>(q);
    P.z = o->z ? o->z : reinterpret_cast<float *>(wsb + L.zbuf);
    P.z_stride = o->z ? sparse->cap : L.z_stride;
    P.sel_len = o->sel_len;
    P.cut = o->cut;
    P.idx = flat ? reinterpret_cast<int32_t *>(wsb + L.idxbuf) : o->idx;
    P.idx_user = o->idx;
    P.offsets = o->offsets;
    P.out = o->out;
    P.lse = o->lse;
    P.m_out = o->m;
    P.logZ_out = o->logZ;
    P.k_out = static_cast<char *>(o->k_out);
    P.v_out = static_cast<char *>(o->v_out);
    const int tickets = P.units * (P.score_tiles + P.attn_tiles);
    s = dispatch<RunStep>(prob, P, tickets, (cudaStream_t)stream);
    if (s != HKV_OK || (!flat && !rewrite))
        return s;
    if (prob->dtype == HKV_BF16)
        return launch(k_flatten<2>, P.units, 0, (cudaStream_t)stream, P);
    return launch(k_flatten<4>, P.units, 0, (cudaStream_t)stream, P);
}

}  // extern "C"
