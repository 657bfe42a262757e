// s6_common.cuh -- device helpers shared by the S6 kernels (sm_100a only).
//
// Transcendentals are issued as the MUFU instructions themselves through PTX
// (ex2.approx / lg2.approx / rcp.approx); every use states the identity it
// relies on.  Bulk tensor copies (TMA) and their mbarriers are plain PTX as
// documented for sm_90+/sm_100.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace s6 {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------- I/O types
template <typename IO>
struct io_traits;

template <>
struct io_traits<float> {
    static __device__ __forceinline__ float to_f(float v) { return v; }
    static __device__ __forceinline__ float from_f(float v) { return v; }
};

template <>
struct io_traits<__nv_bfloat16> {
    // bf16 -> f32 is exact: the bf16 bits are the top half of the f32 bits.
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) {
        return __uint_as_float(static_cast<uint32_t>(__bfloat16_as_ushort(v)) << 16);
    }
    // f32 -> bf16, round to nearest even (cvt.rn.bf16.f32).
    static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// ------------------------------------------------------------- MUFU wrappers
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// SiLU(v) = v * sigmoid(v) = v / (1 + 2^(-v log2 e)).  For v -> -inf the
// power overflows to +inf and the reciprocal to 0, giving -0.
__device__ __forceinline__ float silu_f(float v) {
    return v * rcp_approx(1.0f + ex2_approx(-v * kLog2e));
}

// ------------------------------------------- FMA-pipe function evaluation
// These move work off the special-function (MUFU) pipe, which the decays
// keep busy, onto the FMA pipe.  Coefficients and constants were fitted for
// this library (relative-error least squares on Chebyshev points, float64)
// and checked in float32 Horner evaluation; the bounds are stated per function.

// 1/x for x in [1, 2^120]: exponent-negation seed y0 = bits(K - bits(x))
// (max relative error 5.1e-2 over a binade for K = 0x7EF311C0), then three
// Newton steps y <- y (2 - x y) (error squares each step: < 1e-9 before
// float32 rounding).
__device__ __forceinline__ float rcp_newton(float x) {
    float y = __int_as_float(0x7EF311C0 - __float_as_int(x));
    float e = fmaf(-x, y, 1.0f);
    y = fmaf(y, e, y);
    e = fmaf(-x, y, 1.0f);
    y = fmaf(y, e, y);
    e = fmaf(-x, y, 1.0f);
    return fmaf(y, e, y);
}

// SiLU with one MUFU op: the exponent argument is clamped at 120 so the
// reciprocal stays in the normal range (SiLU(v) < 1e-34 there anyway).
__device__ __forceinline__ float silu_fast(float v) {
    const float e = ex2_approx(fminf(-v * kLog2e, 120.0f));
    return v * rcp_newton(1.0f + e);
}

// ----------------------------------------------------- packed float32 pairs
// sm_100 executes two float32 lanes per instruction (add/mul/fma .f32x2);
// a pair lives in one 64-bit register (low half = first element).
typedef unsigned long long f2_t;

__device__ __forceinline__ f2_t f2_pack(float lo, float hi) {
    f2_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(f2_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f2_t f2_fma(f2_t a, f2_t b, f2_t c) {
    f2_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ f2_t f2_mul(f2_t a, f2_t b) {
    f2_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2_t f2_add(f2_t a, f2_t b) {
    f2_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2_t f2_sub(f2_t a, f2_t b) {
    f2_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// SiLU of a pair: one MUFU ex2 per element, reciprocal by the same seed and
// Newton steps as rcp_newton, in packed arithmetic.
__device__ __forceinline__ f2_t f2_silu_fast(f2_t v) {
    float v0, v1;
    f2_unpack(v, v0, v1);
    const float e0 = ex2_approx(fminf(-v0 * kLog2e, 120.0f));
    const float e1 = ex2_approx(fminf(-v1 * kLog2e, 120.0f));
    const f2_t one = f2_pack(1.0f, 1.0f);
    const f2_t x = f2_add(f2_pack(e0, e1), one);
    float x0, x1;
    f2_unpack(x, x0, x1);
    f2_t y = f2_pack(__int_as_float(0x7EF311C0 - __float_as_int(x0)), __int_as_float(0x7EF311C0 - __float_as_int(x1)));
    const f2_t nx = f2_mul(x, f2_pack(-1.0f, -1.0f));
    f2_t e = f2_fma(nx, y, one);
    y = f2_fma(y, e, y);
    e = f2_fma(nx, y, one);
    y = f2_fma(y, e, y);
    e = f2_fma(nx, y, one);
    y = f2_fma(y, e, y);
    return f2_mul(v, y);
}

__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// SiLU of a pair through the hyperbolic tangent: SiLU(v) = v sigmoid(v) =
// (v/2)(1 + tanh(v/2)), one MUFU op per element and two packed FMA-pipe ops.
// tanh.approx carries a relative error of about 2^-11, below the rounding of a
// bfloat16 output; float32 I/O uses f2_silu_fast instead.
__device__ __forceinline__ f2_t f2_silu_tanh(f2_t v) {
    const f2_t hv = f2_mul(v, f2_pack(0.5f, 0.5f));
    float h0, h1;
    f2_unpack(hv, h0, h1);
    const f2_t t = f2_pack(tanh_approx(h0), tanh_approx(h1));
    return f2_fma(hv, t, hv);
}

// softplus of a pair, softplus(v) = max(v, 0) + log1p(e^-|v|): one MUFU ex2 per
// element for e = e^-|v|, then log1p(e) = e q(e) with q of degree 9 on [0, 1]
// (float32 evaluation: max relative error 1.4e-7) in packed arithmetic.
__device__ __forceinline__ f2_t f2_softplus_fast(f2_t v) {
    float v0, v1;
    f2_unpack(v, v0, v1);
    const f2_t e = f2_pack(ex2_approx(-fabsf(v0) * kLog2e), ex2_approx(-fabsf(v1) * kLog2e));
#define S6_C2(c) f2_pack(c, c)
    f2_t q = S6_C2(-0.0032439918722957373f);
    q = f2_fma(q, e, S6_C2(0.019851312041282654f));
    q = f2_fma(q, e, S6_C2(-0.056959252804517746f));
    q = f2_fma(q, e, S6_C2(0.10603626072406769f));
    q = f2_fma(q, e, S6_C2(-0.15305575728416443f));
    q = f2_fma(q, e, S6_C2(0.19675932824611664f));
    q = f2_fma(q, e, S6_C2(-0.24954132735729218f));
    q = f2_fma(q, e, S6_C2(0.3332996368408203f));
    q = f2_fma(q, e, S6_C2(-0.4999990165233612f));
    q = f2_fma(q, e, S6_C2(1.0f));
#undef S6_C2
    return f2_fma(e, q, f2_pack(fmaxf(v0, 0.0f), fmaxf(v1, 0.0f)));
}

// softplus(v) = log(1 + e^v) = max(v, 0) + log1p(e^-|v|).
// log1p(e) is formed as log2(1 + e) * ln2, corrected for the rounding of
// 1 + e by the factor e / ((1 + e) - 1) (the subtraction is exact); when
// 1 + e rounds to 1, log1p(e) = e to within e^2/2.
__device__ __forceinline__ float softplus_f(float v) {
    const float e = ex2_approx(-fabsf(v) * kLog2e);
    const float u = 1.0f + e;
    const float um1 = u - 1.0f;
    float l = lg2_approx(u) * kLn2;
    l = (um1 == 0.0f) ? e : l * (e * rcp_approx(um1));
    return fmaxf(v, 0.0f) + l;
}

// --------------------------------------------------------- mbarrier + TMA
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
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

// try_wait with a suspend-time hint: the thread may sleep up to `ns`
// nanoseconds (or until the phase completes) instead of returning at once, so a
// warp that waits long issues few instructions.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Bounded wait with suspend hints; at most `limit` polls of at most `ns` each.
__device__ __forceinline__ bool mbar_wait_sleep_bounded(uint64_t *bar, uint32_t parity, uint32_t limit, uint32_t ns) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait_sleep(bar, parity, ns))
            return true;
    return false;
}

// Bounded wait on an mbarrier phase.  Returns false after `limit` polls (each
// try_wait may itself suspend the thread for a short, hardware-chosen time).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity))
            return true;
    return false;
}

// 3-D tiled bulk tensor load global -> shared, completing on `bar`.
// Coordinates are element indices, innermost first; out-of-range elements
// (including negative coordinates of the outer dimensions) are filled with 0.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// 3-D tiled bulk tensor store shared -> global (out-of-range elements are
// not written).  Completion is tracked with bulk groups.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

// Untiled bulk copy global -> shared of `bytes` bytes, completing on `bar`.
// Both addresses 16-byte aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Untiled bulk copy shared -> global of `bytes` bytes, tracked by bulk groups.
// Both addresses 16-byte aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait_group() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (needed before a bulk store reads them).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------- flags between thread blocks
__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(unsigned int *p, unsigned int v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Device-side error word (one per device image of the library; the library is
// built as a single translation unit, s6_abi.cu).  Bit 0: a bounded wait gave
// up.  Read and cleared by the host through s6_device_status.
__device__ unsigned int g_s6_device_error = 0;

__device__ __forceinline__ void raise_device_error(unsigned int bits) { atomicOr(&g_s6_device_error, bits); }

}  // namespace s6
