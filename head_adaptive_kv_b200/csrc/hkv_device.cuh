// hkv_device.cuh -- sm_100a device primitives shared by the HARD-KV kernels:
// mbarrier + bulk-copy (TMA) staging, packed fp32x2 FMA, bf16 widening, warp
// and block reductions, the order key of a score, bounded waits.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "hkv.h"

namespace hkv {

// ---------------------------------------------------------------------------
// CTA shape shared by every kernel: NCW consumer warps and one producer warp.
// The producer issues bulk copies into a ring of NSLOT slots (one per consumer
// warp); the consumers turn staged rows into scores or attention partials.
constexpr int NCW = 4;
constexpr int NSLOT = NCW;
constexpr int NTHREADS = (NCW + 1) * 32;
constexpr int PRODUCER_WARP = NCW;
constexpr int SLOT_BYTES = 16384;
constexpr int SC_FLOATS = 512;  // per-warp logits scratch of an attention stage

// Select histograms: 11 + 11 + 10 bits of the 32-bit order key.
constexpr int L1_BITS = 11, L2_BITS = 11, L3_BITS = 10;
constexpr int HBINS = 1 << 11;

// Calibrated weights exp(beta (z - m)) <= 1 are summed as unsigned fixed-point
// integers with 40 fractional bits: exact, order-free and deterministic.
constexpr int WFIX_BITS = 40;

struct Ctl {
    uint32_t *status;   // device status word (HKV_DEV_* bits)
    uint64_t wait_ns;   // bound of every spin-wait
};

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void raise_flag(const Ctl &c, uint32_t bit) { atomicOr(c.status, bit); }

__device__ __forceinline__ bool timed_out(const Ctl &c)
{
    return (*reinterpret_cast<volatile const uint32_t *>(c.status) & HKV_DEV_TIMEOUT) != 0;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ---------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase of `bar` with the given parity to complete, at most
// c.wait_ns nanoseconds. On expiry the status word gets HKV_DEV_TIMEOUT and
// every later wait in any CTA returns false at once.
__device__ __noinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, const Ctl &c)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 15u) == 0) {
            if (timed_out(c))
                return false;
            if (global_ns() - t0 > c.wait_ns) {
                raise_flag(c, HKV_DEV_TIMEOUT);
                return false;
            }
        }
    }
}

// 1-D bulk copy (TMA) global -> this CTA's shared memory, completing `bytes`
// on `bar`. Both addresses 16-byte aligned, bytes a multiple of 16. Keys and
// values are streamed once per step, so the lines are marked evict-first in L2.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// ---- arithmetic -------------------------------------------------------------

// Two bf16 packed in a 32-bit word widened to two floats (exact).
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w)
{
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// d = a * b + c on a pair of fp32 lanes (one packed sm_100 FMA).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    unsigned long long ra, rb, rc, rd;
    asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(rc) : "f"(c.x), "f"(c.y));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
    float2 d;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
    return d;
}

// Order key of a score: ascending key = descending score; -0 and +0 share one
// key. NaN scores are outside the contract.
__device__ __forceinline__ uint32_t score_key(float z)
{
    uint32_t u = __float_as_uint(z);
    if (u == 0x80000000u)
        u = 0u;
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ~ord;
}

__device__ __forceinline__ float key_score(uint32_t key)
{
    const uint32_t ord = ~key;
    const uint32_t u = (ord & 0x80000000u) ? (ord & 0x7fffffffu) : ~ord;
    return __uint_as_float(u);
}

// Calibrated weight exp(beta (z - m)) in fixed point (1.0 = 2^40); exactly 1.0
// at the maximum and everywhere when beta = 0.
__device__ __forceinline__ unsigned long long wfix(float z, float m, float beta)
{
    if (z == m || beta == 0.0f)
        return 1ull << WFIX_BITS;
    const float w = expf(beta * (z - m));
    return __float2ull_rn(w * 1099511627776.0f);
}

// ---- warp / block reductions ------------------------------------------------

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Exclusive prefix sum over the CTA (NTHREADS threads) of a 64-bit value.
// `scratch` holds at least NTHREADS/32 + 1 words. *total receives the sum.
// Contains __syncthreads(); every thread must call it.
__device__ __forceinline__ unsigned long long block_exclusive_scan(unsigned long long v,
                                                                   unsigned long long *scratch,
                                                                   unsigned long long *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NW = NTHREADS / 32;
    unsigned long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o)
            x += y;
    }
    if (lane == 31)
        scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        unsigned long long w = lane < NW ? scratch[lane] : 0ull;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o)
                w += y;
        }
        if (lane < NW)
            scratch[lane] = w;  // inclusive prefix over warps
    }
    __syncthreads();
    const unsigned long long before_warp = warp > 0 ? scratch[warp - 1] : 0ull;
    *total = scratch[NW - 1];
    __syncthreads();
    return before_warp + x - v;
}

__device__ __forceinline__ float block_max(float v, float *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NW = NTHREADS / 32;
    v = warp_max(v);
    if (lane == 0)
        scratch[warp] = v;
    __syncthreads();
    float r = scratch[0];
#pragma unroll
    for (int i = 1; i < NW; ++i)
        r = fmaxf(r, scratch[i]);
    __syncthreads();
    return r;
}

__device__ __forceinline__ unsigned long long block_sum_u64(unsigned long long v, unsigned long long *scratch)
{
    unsigned long long total;
    block_exclusive_scan(v, scratch, &total);
    return total;
}

// Acquire / release flags between CTAs (published selections).
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(uint32_t *p, uint32_t v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

}  // namespace hkv
