// Device primitives shared by the ParaRNN kernels: PTX wrappers for mbarriers,
// TMA tensor loads, a grid barrier, bounded waits, bf16 unpacking and the
// elementary functions the cells need.
//
// Every wait here is bounded: it gives up after a time limit (read from the
// %globaltimer register), records an error code in device memory and returns
// false, so a kernel never spins forever.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pararnn_internal.h"

namespace pararnn {

// ------------------------------------------------------------------ PTX basics

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned ld_acquire_gpu_u32(const unsigned* p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ int ld_relaxed_gpu(const int* p)
{
    int v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add_gpu(unsigned* p, unsigned v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Orders this thread's earlier generic-proxy view of global memory before its
// later async-proxy (TMA) reads.
__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_shared()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_inval(uint64_t* bar)
{
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
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

// try_wait with a suspend-time hint: the warp is parked (issuing nothing) until
// the phase completes or about `hint_ns` nanoseconds pass, so a waiting warp
// does not take issue slots from the warps doing the arithmetic.
__device__ __forceinline__ bool mbar_try_wait_parked(uint64_t* bar, uint32_t parity, uint32_t hint_ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Longest single park of a bounded wait (ns); the time limit is checked
// between parks.
constexpr uint32_t kParkNs = 200000u;

// ------------------------------------------------------------------------ TMA
// Tiled bulk tensor loads into this CTA's shared memory, completing on an
// mbarrier.  No multicast.

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int c0, int c1, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
        "l"(tm), "r"(c0), "r"(c1), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, int c0, int c1, int c2,
                                            uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
        "l"(tm), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* tm, int c0, int c1, int c2,
                                            int c3, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_addr(dst)),
        "l"(tm), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* tm)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(tm) : "memory");
}

// --------------------------------------------------------------- error flags

__device__ __forceinline__ void raise_error(int* err, int code)
{
    atomicCAS(err, 0, code);
}

__device__ __forceinline__ bool error_raised(const int* err)
{
    return ld_relaxed_gpu(err) != 0;
}

// Waits for this CTA's TMA transaction on `bar` (phase `parity`).  Bounded.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* err,
                                                  uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        if (mbar_try_wait_parked(bar, parity, kParkNs)) return true;
        if (global_timer_ns() - t0 > limit_ns) {
            raise_error(err, PARARNN_ERR_TIMEOUT);
            return false;
        }
    }
}

// Grid-wide barrier for a cooperative launch (all CTAs co-resident).
// `counter` increases monotonically; generation g completes when it reaches
// (g+1)*gridDim.x.  Bounded: on timeout raises PARARNN_ERR_TIMEOUT and
// returns false.  Must be called by every thread of the CTA.
__device__ __forceinline__ bool grid_barrier(unsigned* counter, unsigned generation, int* err,
                                             uint64_t limit_ns, int* s_flag)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        __threadfence();
        red_release_add_gpu(counter, 1u);
        const unsigned target = (generation + 1u) * gridDim.x;
        uint64_t t0 = 0;
        for (unsigned n = 0;; ++n) {
            if (ld_acquire_gpu_u32(counter) >= target) break;
            if ((n & 31u) == 31u) {
                uint64_t now = global_timer_ns();
                if (t0 == 0) {
                    t0 = now;
                } else if (now - t0 > limit_ns) {
                    raise_error(err, PARARNN_ERR_TIMEOUT);
                    ok = 0;
                    break;
                }
            }
            if (n >= 16) __nanosleep(128);
        }
        __threadfence();
        *s_flag = ok;
    }
    __syncthreads();
    return *s_flag != 0;
}

// ------------------------------------------------------------------ bf16 / u

struct F4 {
    float v[4];
};

// Four consecutive channels of one gate row, from bf16 (8 bytes) or fp32.
__device__ __forceinline__ F4 load4(const uint16_t* p)
{
    uint2 w = *reinterpret_cast<const uint2*>(p);
    F4 r;
    r.v[0] = __uint_as_float(w.x << 16);
    r.v[1] = __uint_as_float(w.x & 0xffff0000u);
    r.v[2] = __uint_as_float(w.y << 16);
    r.v[3] = __uint_as_float(w.y & 0xffff0000u);
    return r;
}

__device__ __forceinline__ F4 load4(const float* p)
{
    float4 w = *reinterpret_cast<const float4*>(p);
    F4 r;
    r.v[0] = w.x;
    r.v[1] = w.y;
    r.v[2] = w.z;
    r.v[3] = w.w;
    return r;
}

// N = 4 or 2 consecutive values (16- or 8-byte accesses; bf16 widened).
template <int N>
struct FV {
    float v[N];
};

template <int N>
__device__ __forceinline__ FV<N> loadv(const float* p)
{
    FV<N> r;
    if constexpr (N == 4) {
        const float4 w = *reinterpret_cast<const float4*>(p);
        r.v[0] = w.x;
        r.v[1] = w.y;
        r.v[2] = w.z;
        r.v[3] = w.w;
    } else {
        static_assert(N == 2, "2 or 4 values");
        const float2 w = *reinterpret_cast<const float2*>(p);
        r.v[0] = w.x;
        r.v[1] = w.y;
    }
    return r;
}

template <int N>
__device__ __forceinline__ FV<N> loadv(const uint16_t* p)
{
    FV<N> r;
    if constexpr (N == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(p);
        r.v[0] = __uint_as_float(w.x << 16);
        r.v[1] = __uint_as_float(w.x & 0xffff0000u);
        r.v[2] = __uint_as_float(w.y << 16);
        r.v[3] = __uint_as_float(w.y & 0xffff0000u);
    } else {
        static_assert(N == 2, "2 or 4 values");
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
        r.v[0] = __uint_as_float(w << 16);
        r.v[1] = __uint_as_float(w & 0xffff0000u);
    }
    return r;
}

template <int N>
__device__ __forceinline__ void storev(float* p, const float* v)
{
    if constexpr (N == 4) *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
}

// streaming store to global memory (kept in L2 only)
template <int N>
__device__ __forceinline__ void stcgv(float* p, const float* v)
{
    if constexpr (N == 4) __stcg(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    else __stcg(reinterpret_cast<float2*>(p), make_float2(v[0], v[1]));
}

__device__ __forceinline__ void store4(float* p, const float* v)
{
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

// --------------------------------------------------------- elementary math
//
// The gates need e^x and 1/x.  Both use the special-function unit: ex2.approx
// (2^x, at most 2 ulp) and rcp.approx (at most 1 ulp) from the PTX ISA.  The
// logistic function and tanh are written from their definitions:
//   s(x) = 1 / (1 + e^-x),   tanh(x) = 1 - 2 / (1 + e^(2x)),
// with e^y = 2^(y log2 e).  Two logistic denominators share one reciprocal:
// 1/d1 = d2 / (d1 d2) and 1/d2 = d1 / (d1 d2); the exponents are clamped from
// above at kMaxT so that d1 d2 < 2^121 stays finite (the clamp changes s(x)
// only for s(x) < 2^-60).  NaN arguments give NaN results (the clamp is the
// NaN-keeping min).

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kMaxT = 60.0f;

__device__ __forceinline__ float ex2_approx(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float rcp_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float min_keep_nan(float x, float hi)
{
    float r;
    asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(x), "f"(hi));
    return r;
}

// max(a, b) with NaN kept (either NaN gives NaN)
__device__ __forceinline__ float max_keep_nan(float a, float b)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// 1 + e^-x with the exponent clamped (see above)
__device__ __forceinline__ float logistic_den(float x)
{
    return 1.0f + ex2_approx(min_keep_nan(-kLog2e * x, kMaxT));
}

// 1 + e^(2x) with the exponent clamped (see above)
__device__ __forceinline__ float tanh_den(float x)
{
    return 1.0f + ex2_approx(min_keep_nan(2.0f * kLog2e * x, kMaxT));
}

// s(x), s(y) with one reciprocal
__device__ __forceinline__ void sigmoid2(float x, float y, float& sx, float& sy)
{
    const float dx = logistic_den(x), dy = logistic_den(y);
    const float inv = rcp_approx(dx * dy);
    sx = dy * inv;
    sy = dx * inv;
}

// s(x), tanh(y) with one reciprocal
__device__ __forceinline__ void sigmoid_tanh(float x, float y, float& sx, float& ty)
{
    const float dx = logistic_den(x), dy = tanh_den(y);
    const float inv = rcp_approx(dx * dy);
    sx = dy * inv;
    ty = fmaf(-2.0f * dx, inv, 1.0f);
}

__device__ __forceinline__ float tanh_fast(float x)
{
    return fmaf(-2.0f, rcp_approx(1.0f + ex2_approx(2.0f * kLog2e * x)), 1.0f);
}

}  // namespace pararnn
