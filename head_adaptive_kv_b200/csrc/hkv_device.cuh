// hkv_device.cuh -- sm_100a device primitives shared by the HARD-KV kernels:
// mbarriers, bulk copies (TMA) and cp.async, packed fp32x2 FMA, bf16
// widening, warp and block reductions, the order key of a score, the
// fixed-point calibrated weight, bounded waits and an optional device trace.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "hkv.h"

namespace hkv {

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

// Optional device trace (build with -DHKV_TRACE): thread 0 of a CTA (or lane 0
// of a warp, HKV_TRACE_WARP) stores the global timer at a numbered slot.
#ifdef HKV_TRACE
constexpr int HKV_TRACE_SLOTS = 1 << 18;
__device__ unsigned long long hkv_trace_buf[HKV_TRACE_SLOTS];  // one translation unit per trace build
#define HKV_TRACE_IF(cond, slot)                                                   \
    do {                                                                           \
        const int hkv_slot_ = (slot);                                              \
        if ((cond) && hkv_slot_ >= 0 && hkv_slot_ < HKV_TRACE_SLOTS)               \
            hkv_trace_buf[hkv_slot_] = global_ns();                                \
    } while (0)
#define HKV_TRACE_VAL(slot, v)                                                     \
    do {                                                                           \
        const int hkv_slot_ = (slot);                                              \
        if (threadIdx.x == 0 && hkv_slot_ >= 0 && hkv_slot_ < HKV_TRACE_SLOTS)     \
            hkv_trace_buf[hkv_slot_] = (unsigned long long)(v);                    \
    } while (0)
#else
#define HKV_TRACE_IF(cond, slot) \
    do {                         \
    } while (0)
#define HKV_TRACE_VAL(slot, v) \
    do {                       \
    } while (0)
#endif
#define HKV_TRACE_AT(slot) HKV_TRACE_IF(threadIdx.x == 0, slot)
#define HKV_TRACE_WARP(slot) HKV_TRACE_IF((threadIdx.x & 31) == 0, slot)

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

// Non-blocking test of a phase.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Slow path of mbar_wait: spin at most wait_ns nanoseconds. On expiry the
// status word gets HKV_DEV_TIMEOUT and every later wait in any CTA returns
// false at once.
__device__ __noinline__ bool mbar_wait_slow(uint64_t *bar, uint32_t parity, uint32_t *status, uint64_t wait_ns)
{
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 15u) == 0) {
            if ((*reinterpret_cast<volatile const uint32_t *>(status) & HKV_DEV_TIMEOUT) != 0)
                return false;
            if (global_ns() - t0 > wait_ns) {
                atomicOr(status, HKV_DEV_TIMEOUT);
                return false;
            }
        }
    }
}

// Wait at most wait_ns for the phase of `bar` with the given parity, whatever
// the status word says (used to let copies already started land before a CTA
// exits after a timeout).
__device__ __noinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t wait_ns)
{
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 15u) == 0 && global_ns() - t0 > wait_ns)
            return false;
    }
}

// Wait for the phase of `bar` with the given parity to complete (bounded).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, const Ctl &c)
{
    if (mbar_try_wait(bar, parity))
        return true;
    return mbar_wait_slow(bar, parity, c.status, c.wait_ns);
}

// ---- copies -------------------------------------------------------------------

// 1-D bulk copy (TMA) global -> this CTA's shared memory, completing `bytes`
// on `bar`. Both addresses 16-byte aligned, bytes a multiple of 16. Keys and
// values are streamed once per step, so the lines are marked evict-first.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// Four rows of a 2-D tensor map whose box is one row high (row0 .. row3, from
// column 0), gathered by the TMA into dst one after another; completion is
// counted in bytes on bar. No multicast.
__device__ __forceinline__ void tma_gather4(void *dst, const CUtensorMap *map, int r0, int r1, int r2, int r3,
                                            uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_addr(bar))
        : "memory");
}

// 16-byte asynchronous copy global -> shared, cached in L2 only.
__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

// Wait until this thread's earlier cp.async copies have landed (a barrier
// then makes every thread's copies visible to the CTA).
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Arrive on `bar` once this thread's earlier cp.async copies have landed (the
// pending count is raised first, so the phase waits for them).
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Order earlier ordinary (generic-proxy) shared-memory accesses before later
// bulk copies (async proxy) into the same memory.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint64_t evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Programmatic dependent launch: wait for the preceding kernel's results
// (its completion and the visibility of its writes).
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Let the next kernel on the stream, if launched as a programmatic dependent,
// start its CTAs now; it still waits for this grid's completion before it
// reads anything this grid writes.
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- shared-memory accesses with an explicit state space ----------------------
// (functions that receive shared memory through a reference cannot always
// prove it is shared, and would otherwise use slower generic accesses)

__device__ __forceinline__ void sred_add(uint32_t *p, uint32_t v)
{
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(smem_addr(p)), "r"(v) : "memory");
}
__device__ __forceinline__ void sred_add(unsigned long long *p, unsigned long long v)
{
    asm volatile("red.shared.add.u64 [%0], %1;" ::"r"(smem_addr(p)), "l"(v) : "memory");
}
__device__ __forceinline__ int satom_add(int *p, int v)
{
    int old;
    asm volatile("atom.shared.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_addr(p)), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ float4 lds4(const float *p)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(smem_addr(p))
                 : "memory");
    return v;
}
__device__ __forceinline__ float lds1(const float *p)
{
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(smem_addr(p)) : "memory");
    return v;
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

// 2^x on the SFU (ex2.approx, relative error below 2^-22).
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Calibrated weight exp(beta (z - m)) = 2^((z - m) beta log2 e), exactly 1 at
// the maximum and everywhere when beta = 0. bl2 = beta * log2(e). Its relative
// error is below 2^-22 (ex2.approx) + 3 2^-24 ln2 |x|, x = (z - m) beta log2 e,
// the second term from the three fp32 roundings of the exponent.
__device__ __forceinline__ float wcal(float z, float m, float bl2)
{
    if (z == m || bl2 == 0.0f)
        return 1.0f;
    return ex2((z - m) * bl2);
}

// floor(w * 2^40) of a weight 0 <= w <= 1, from its bits (exact integer ops):
// w = mant * 2^(e - 23) with a 24-bit mant, so w * 2^40 = mant * 2^(e + 17).
__device__ __forceinline__ unsigned long long wq(float w)
{
    const uint32_t bits = __float_as_uint(w);
    const int e = (int)((bits >> 23) & 0xffu) - 127;
    if (e < -41)  // below 2^-41 (including 0 and subnormals) contributes nothing
        return 0ull;
    const unsigned long long mant = (unsigned long long)((bits & 0x7fffffu) | 0x800000u);
    const int sh = e + 17;
    return sh >= 0 ? (mant << sh) : (mant >> (-sh));
}

// Calibrated weight in fixed point (1.0 = 2^WFIX_BITS).
__device__ __forceinline__ unsigned long long wfix(float z, float m, float bl2) { return wq(wcal(z, m, bl2)); }

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

// Exclusive prefix sum over a CTA of NT threads of a 64-bit value. `scratch`
// holds at least NT/32 words. *total receives the sum. Contains
// __syncthreads(); every thread must call it.
template <int NT>
__device__ __forceinline__ unsigned long long block_exclusive_scan(unsigned long long v, unsigned long long *scratch,
                                                                   unsigned long long *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NW = NT / 32;
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

template <int NT>
__device__ __forceinline__ unsigned long long block_sum_u64(unsigned long long v, unsigned long long *scratch)
{
    unsigned long long total;
    block_exclusive_scan<NT>(v, scratch, &total);
    return total;
}

template <int NT>
__device__ __forceinline__ float block_max(float v, float *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NW = NT / 32;
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

}  // namespace hkv
