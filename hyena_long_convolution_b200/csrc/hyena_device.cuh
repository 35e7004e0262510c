// hyena_device.cuh -- device-side helpers shared by the sm_100a kernels:
// mbarrier + TMA (cp.async.bulk.tensor) staging, acquire/release flag access,
// bounded waits, bf16x2 packing.  Hand-written inline PTX; no library code.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hyena {

// Error bits recorded in a workspace header word by bounded waits.
enum : unsigned int {
    kErrLookbackTimeout = 1u,
    kErrTmaTimeout = 2u,
    kErrRingTimeout = 4u,
    kErrLocalTimeout = 8u,  // a hand-off between a CTA's own warps ran out
};

// A bounded wait gives up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test: true if the phase with the given parity has completed.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete; false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    }
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 3-D tiled TMA load (no multicast) into this CTA's shared memory; completion
// is signalled on `bar` as transaction bytes.  c0 is the innermost (channel)
// coordinate and must be a multiple of 8 bf16 elements (16 bytes).
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// 4-D tiled TMA load (no multicast), as tma_load_3d with one more coordinate.
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2, int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}

// 2-D tiled TMA load (no multicast); c0 is the innermost coordinate and must
// be 16-byte aligned in bytes.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// ---------------------------------------------------------------- flags

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned int ld_volatile_u32(const unsigned int *p)
{
    unsigned int v;
    asm volatile("ld.volatile.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// ---------------------------------------------------------------- bf16

// Two bf16 values packed in one 32-bit word (low half = lower channel) to two
// fp32 values; exact.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w)
{
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Per-channel triples (x1_c, x2_c, x3_c adjacent): a channel pair (c, c+1)
// occupies six bf16 values, x1_c x2_c x3_c x1_{c+1} x2_{c+1} x3_{c+1}, read as
// three words w0 w1 w2 (lower address = low half).  Each helper returns the
// pair (value of c, value of c+1) of one input; exact.
__device__ __forceinline__ float2 tri_x1(uint32_t w0, uint32_t w1)
{
    return make_float2(__uint_as_float(w0 << 16), __uint_as_float(w1 & 0xffff0000u));
}
__device__ __forceinline__ float2 tri_x2(uint32_t w0, uint32_t w2)
{
    return make_float2(__uint_as_float(w0 & 0xffff0000u), __uint_as_float(w2 << 16));
}
__device__ __forceinline__ float2 tri_x3(uint32_t w1, uint32_t w2)
{
    return make_float2(__uint_as_float(w1 << 16), __uint_as_float(w2 & 0xffff0000u));
}

// Two fp32 values to two bf16 (round to nearest even), packed low = .x.
__device__ __forceinline__ uint32_t float2_to_bf16x2(float2 f)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<uint32_t *>(&h);
}

// ---------------------------------------------------------------- modal modes
// A lane's state of NP mode slots for its channel pair.  Real modes: slot n is
// mode n.  Complex modes (pole p = pr + i pi): slots 2m and 2m+1 hold the real
// and imaginary parts of mode m, of the state as of the pole.

// One token, s <- p s + v with real v (packed f32x2 over the channel pair).
template <int NP, bool kCx>
__device__ __forceinline__ void modes_step(float2 (&s)[NP], const float2 (&p)[NP], float2 v)
{
    if constexpr (!kCx) {
#pragma unroll
        for (int n = 0; n < NP; ++n) s[n] = __ffma2_rn(p[n], s[n], v);
    } else {
#pragma unroll
        for (int m = 0; m < NP; m += 2) {
            const float2 re = s[m], im = s[m + 1];
            const float2 npi = make_float2(-p[m + 1].x, -p[m + 1].y);
            s[m] = __ffma2_rn(p[m], re, __ffma2_rn(npi, im, v));
            s[m + 1] = __ffma2_rn(p[m], im, __fmul2_rn(p[m + 1], re));
        }
    }
}

// One carry step of a slot pair (two real modes, or the real and imaginary
// slots of one complex mode), C <- P C + A with a full state A (P = p^k).
template <bool kCx>
__device__ __forceinline__ void carry_pair(float2 &c0, float2 &c1, float2 P0, float2 P1, float2 A0, float2 A1)
{
    if constexpr (!kCx) {
        c0 = __ffma2_rn(P0, c0, A0);
        c1 = __ffma2_rn(P1, c1, A1);
    } else {
        const float2 re = c0, im = c1;
        const float2 npi = make_float2(-P1.x, -P1.y);
        c0 = __ffma2_rn(P0, re, __ffma2_rn(npi, im, A0));
        c1 = __ffma2_rn(P0, im, __ffma2_rn(P1, re, A1));
    }
}

// One carry step of all NP slots, C <- P C + A (the same operations as
// carry_pair on each slot pair).
template <int NP, bool kCx>
__device__ __forceinline__ void modes_carry(float2 (&C)[NP], const float2 (&P)[NP], const float2 (&A)[NP])
{
#pragma unroll
    for (int m = 0; m < NP; m += 2) carry_pair<kCx>(C[m], C[m + 1], P[m], P[m + 1], A[m], A[m + 1]);
}

__device__ __forceinline__ float2 ldg_f2(const float *p)
{
    return __ldg(reinterpret_cast<const float2 *>(p));
}

// Same load, but never merged with another load of the same address: keeps
// per-phase coefficient copies from being held in registers across phases.
__device__ __forceinline__ float2 ldg_f2_fresh(const float *p)
{
    float2 v;
    asm volatile("ld.global.nc.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
    return v;
}

}  // namespace hyena
