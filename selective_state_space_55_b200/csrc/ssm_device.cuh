// Device helpers shared by the scan and update kernels (sm_100a).
//
//  - PTX wrappers: mbarrier, TMA tensor loads, MUFU ex2, proxy fences.
//  - softplus and silu in fp32.
//  - bf16 <-> fp32 packing.
//  - the library's device status word (bounded waits report through it).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mamba_ssm.h"

namespace mamba {

constexpr float kLog2e = 1.4426950408889634f;   // log2(e)
constexpr float kLn2 = 0.6931471805599453f;     // ln(2)
constexpr int kNPad = 16;                        // compiled state size (smaller N is zero-padded)

// First device-side error since the host last read it (0 = none).  The
// library is compiled as one translation unit, which owns this definition.
__device__ int g_device_status = 0;

__device__ __forceinline__ void record_device_error(int code) {
    atomicCAS(&g_device_status, 0, code);
}

// ---------------------------------------------------------------- MUFU / math

// 2^x on the MUFU pipe (ex2.approx, flush-to-zero).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x with unbiased rounding near x = 0.  For |x| < 1/16 the Taylor series
// 1 + x ln2 + (x ln2)^2/2! + (x ln2)^3/3! + (x ln2)^4/4! (truncation below
// 1.3e-9) is evaluated with FMAs whose final rounding is to nearest; elsewhere
// MUFU ex2 is used.  A decay factor Abar = 2^x close to 1 is applied over
// about 1/|x| consecutive steps, so a systematic rounding bias of the hardware
// approximation would grow linearly with that memory length; the series keeps
// the per-step error unbiased, and the error of the product grows only as a
// random walk.
__device__ __forceinline__ float exp2_near_one_exact(float x) {
    constexpr float c1 = 0.6931471805599453f;     // ln 2
    constexpr float c2 = 0.2402265069591007f;     // (ln 2)^2 / 2
    constexpr float c3 = 0.05550410866482158f;    // (ln 2)^3 / 6
    constexpr float c4 = 0.009618129107628477f;   // (ln 2)^4 / 24
    const float series = fmaf(x, fmaf(x, fmaf(x, fmaf(x, c4, c3), c2), c1), 1.0f);
    const float hw = ex2_approx(x);
    return fabsf(x) < 0.0625f ? series : hw;
}

// exp2_near_one_exact on both halves of x, the series in packed fp32x2.
__device__ __forceinline__ float2 exp2_near_one_exact2(float2 x) {
    const float2 c1 = make_float2(0.6931471805599453f, 0.6931471805599453f);
    const float2 c2 = make_float2(0.2402265069591007f, 0.2402265069591007f);
    const float2 c3 = make_float2(0.05550410866482158f, 0.05550410866482158f);
    const float2 c4 = make_float2(0.009618129107628477f, 0.009618129107628477f);
    const float2 one = make_float2(1.0f, 1.0f);
    const float2 series = __ffma2_rn(x, __ffma2_rn(x, __ffma2_rn(x, __ffma2_rn(x, c4, c3), c2), c1), one);
    return make_float2(fabsf(x.x) < 0.0625f ? series.x : ex2_approx(x.x),
                       fabsf(x.y) < 0.0625f ? series.y : ex2_approx(x.y));
}

// Zero-order-hold input gain.  For the diagonal A the exact discretisation
// Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B gives, per state entry,
// Bbar_n = Delta phi(Delta A_n) B_n with phi(x) = (e^x - 1) / x, phi(0) = 1.
// Written in x2 = x log2(e) (the exponent the scan already forms for Abar):
// near 0, phi = 1 + x/2 + x^2/6 + x^3/24 + x^4/120 (truncation below 2.3e-10
// for |x2| < 1/16), which avoids the cancellation in e^x - 1; elsewhere
// phi = (Abar - 1) / x.
constexpr float kZohSmall = 0.0625f;   // |x2| below which the series is used

__device__ __forceinline__ float zoh_phi_series(float x2) {
    constexpr float k1 = 0.34657359027997264f;     // ln2 / 2
    constexpr float k2 = 0.08007550231970023f;     // ln2^2 / 6
    constexpr float k3 = 0.013876027166205394f;    // ln2^3 / 24
    constexpr float k4 = 0.0019236258215256953f;   // ln2^4 / 120
    return fmaf(x2, fmaf(x2, fmaf(x2, fmaf(x2, k4, k3), k2), k1), 1.0f);
}

// zoh_phi_series on both halves, in packed fp32x2.
__device__ __forceinline__ float2 zoh_phi_series2(float2 x2) {
    const float2 k1 = make_float2(0.34657359027997264f, 0.34657359027997264f);
    const float2 k2 = make_float2(0.08007550231970023f, 0.08007550231970023f);
    const float2 k3 = make_float2(0.013876027166205394f, 0.013876027166205394f);
    const float2 k4 = make_float2(0.0019236258215256953f, 0.0019236258215256953f);
    const float2 one = make_float2(1.0f, 1.0f);
    return __ffma2_rn(x2, __ffma2_rn(x2, __ffma2_rn(x2, __ffma2_rn(x2, k4, k3), k2), k1), one);
}

// phi for one entry given x2 = Delta A log2(e) and Abar = 2^x2 (scalar path).
__device__ __forceinline__ float zoh_phi(float x2, float abar) {
    return fabsf(x2) < kZohSmall ? zoh_phi_series(x2) : (abar - 1.0f) / (x2 * kLn2);
}

// softplus(s) = log(1 + e^s) = max(s, 0) + log1p(e^-|s|).
// log1p(w) for w = e^-|s| in (0, 1] is evaluated as 2 atanh(r) with
// r = w / (2 + w) in (0, 1/3]:  2 atanh(r) = 2 r (1 + r^2/3 + r^4/5 + ...).
// Seven terms bring the truncation below 2e-8 relative at r = 1/3, so the
// result keeps fp32 accuracy even where e^-|s| is tiny (where log(1 + w)
// through a hardware log would lose most of its digits).
__device__ __forceinline__ float softplus_f32(float s) {
    const float w = ex2_approx(-fabsf(s) * kLog2e);
    const float r = __fdividef(w, 2.0f + w);
    const float r2 = r * r;
    float p = 1.0f / 13.0f;
    p = fmaf(p, r2, 1.0f / 11.0f);
    p = fmaf(p, r2, 1.0f / 9.0f);
    p = fmaf(p, r2, 1.0f / 7.0f);
    p = fmaf(p, r2, 1.0f / 5.0f);
    p = fmaf(p, r2, 1.0f / 3.0f);
    p = fmaf(p, r2, 1.0f);
    return fmaxf(s, 0.0f) + 2.0f * r * p;
}

// silu(z) = z * sigmoid(z) = z / (1 + e^-z).  For z -> -inf the denominator
// becomes +inf and the result is -0.
__device__ __forceinline__ float silu_f32(float z) {
    return __fdividef(z, 1.0f + ex2_approx(-z * kLog2e));
}

// ---- shorter forms for bf16 inputs and outputs ----------------------------
// The scan is bounded by instruction issue and the MUFU pipe, not by memory,
// so each instruction per step counts.  With bf16 inputs the inputs already
// carry a relative rounding of 2^-9 (for delta near -9 that alone moves Delta
// by about 2%), so these forms trade digits that bf16 cannot hold:
//  - softplus_lg2: log1p(w) = log2(1 + w) ln 2 on MUFU lg2.  1 + w rounds
//    to fp32 and lg2.approx has an absolute error near 2^-22, so Delta is off
//    by at most ~3e-7 absolute (relative ~3e-3 at the smallest Delta ~1e-4 of
//    the layer workloads), against ~16 instructions and an rcp for softplus_f32.
//  - silu_tanh: sigmoid(z) = (1 + tanh(z/2)) / 2, one MUFU tanh (relative
//    error 2^-11) instead of ex2 and rcp; silu is off by at most ~2.5e-4 |z|.
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float softplus_lg2(float s) {
    const float w = ex2_approx(-fabsf(s) * kLog2e);
    return fmaf(lg2_approx(1.0f + w), kLn2, fmaxf(s, 0.0f));
}

__device__ __forceinline__ float silu_tanh(float z) {
    const float hz = 0.5f * z;
    return fmaf(hz, tanh_approx(hz), hz);
}

// ------------------------------------------------------------------- dtypes

template <typename T> struct DType;
template <> struct DType<float> {
    static constexpr int kBytes = 4;
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct DType<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// 16 bytes -> 4 fp32 or 8 bf16 values as fp32.
__device__ __forceinline__ void unpack16(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
}
__device__ __forceinline__ void unpack16(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ uint4 pack16(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint4 pack16(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}

// ------------------------------------------------------------- shared / TMA

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Upper bound on try_wait polls before a wait is declared stuck.  Each poll
// may suspend the thread for a hardware-defined interval; 2^22 polls is far
// beyond any legitimate TMA latency, and still ends in seconds.
constexpr uint32_t kMaxWaitPolls = 1u << 22;

__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kMaxWaitPolls; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// 3-D tiled TMA load into this CTA's shared memory, completing on `bar`.
// c0 is the innermost coordinate (time), c1 the row (channel or state index),
// c2 the batch index.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

// 1-D bulk copy shared -> global, tracked by the issuing thread's bulk groups.
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(reinterpret_cast<uint64_t>(dst)), "r"(src), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N of this thread's committed bulk stores still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until at most N of this thread's committed bulk stores are incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Programmatic dependent launch.  grid_dependency_wait returns once the
// kernels this grid was launched to overlap with have completed and their
// memory is visible (at once when it was launched without that attribute);
// grid_launch_dependents lets the next such kernel on the stream start.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

}  // namespace mamba
