// Single-token selective state update (generation) kernel (sm_100a).
//
// One step of the recurrence applied to a stored state, which is read and
// written in place ("Mamba: Linear-Time Sequence Modeling with Selective State
// Spaces", table 复杂度对比: per-token cost independent of the context length;
// "Mamba 与状态空间模型", section 固定大小的状态: the state keeps its size).
//
// The step is HBM-bound: for N = 16 every chain reads and writes 64 bytes of
// fp32 state against a few bytes of token inputs.  The fast path (N = 16,
// 16-byte aligned state, A, B, C) gives each chain four consecutive lanes;
// lane q loads the float4 of states 4q..4q+3, so a warp streams 512
// contiguous bytes per access, and the four partial readouts are summed with
// two shuffles.  Each thread carries kUpdateItems chains to keep enough bytes
// in flight.  The generic path (any N <= 16, any alignment) uses one thread
// per chain.  Abar uses exp2_near_one_exact: the state persists across calls,
// so an unbiased decay matters over many generated tokens, and this
// memory-bound kernel has ALU time to spare.
#pragma once

#include "ssm_device.cuh"

namespace mamba {

struct UpdateParams {
    float* state;
    const void* x;
    const void* dt;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const void* z;
    const float* dt_bias;
    void* out;
    int64_t batch, dim, chains;
    int dstate;
    int dt_softplus;
};

constexpr int kUpdateThreads = 256;

template <typename T>
__device__ __forceinline__ float load_as_float(const void* base, int64_t i) {
    return DType<T>::load(static_cast<const T*>(base) + i);
}

// Four consecutive (b, n-quarter) values of B or C as fp32.
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 t = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(t.x << 16); v[1] = __uint_as_float(t.x & 0xffff0000u);
    v[2] = __uint_as_float(t.y << 16); v[3] = __uint_as_float(t.y & 0xffff0000u);
}

// Channels handled per thread: each is an independent 16-byte state load, so
// every thread keeps kUpdateItems loads in flight.
#ifndef MAMBA_UPDATE_ITEMS
#define MAMBA_UPDATE_ITEMS 2
#endif
constexpr int kUpdateItems = MAMBA_UPDATE_ITEMS;
constexpr int kUpdateChainsPerCta = (kUpdateThreads / 32) * 8 * kUpdateItems;

// Fast path, N = 16.  blockIdx.y is the batch row (grid-strided), blockIdx.x a
// block of kUpdateChainsPerCta channels.  Item `it` of warp w covers channels
// w*8*kUpdateItems + it*8 .. +7 of the block; lane l owns quarter q = l & 3 of
// channel (l >> 2), so each item is one fully coalesced 512-byte warp access
// of the state.
template <typename IoT, typename BcT, bool kHasZ>
__global__ void __launch_bounds__(kUpdateThreads)
    state_update_n16_kernel(const __grid_constant__ UpdateParams p) {
    const int lane = threadIdx.x & 31;
    const int q = lane & 3;
    const int64_t d_base = (int64_t)blockIdx.x * kUpdateChainsPerCta +
                           (threadIdx.x >> 5) * (8 * kUpdateItems) + (lane >> 2);
    for (int64_t b = blockIdx.y; b < p.batch; b += gridDim.y) {
    bool live[kUpdateItems];
    int64_t dd[kUpdateItems];
    float4 hs[kUpdateItems];
#pragma unroll
    for (int it = 0; it < kUpdateItems; ++it) {
        const int64_t d = d_base + 8 * it;
        live[it] = d < p.dim;
        dd[it] = live[it] ? d : 0;
        hs[it] = __ldcs(reinterpret_cast<float4*>(p.state + (b * p.dim + dd[it]) * 16) + q);
    }
#pragma unroll
    for (int it = 0; it < kUpdateItems; ++it) {
        const int64_t d = dd[it];
        const int64_t c = b * p.dim + d;
        const float4 av = *(reinterpret_cast<const float4*>(p.A + d * 16) + q);
        float Bv[4], Cv[4];
        load4(static_cast<const BcT*>(p.B) + b * 16 + 4 * q, Bv);
        load4(static_cast<const BcT*>(p.C) + b * 16 + 4 * q, Cv);
        const float x = load_as_float<IoT>(p.x, c);
        float s = load_as_float<IoT>(p.dt, c);
        if (p.dt_bias != nullptr) s += p.dt_bias[d];
        const float delta = p.dt_softplus ? softplus_f32(s) : s;
        const float dx = delta * x;

        const float a[4] = {av.x, av.y, av.z, av.w};
        float h[4] = {hs[it].x, hs[it].y, hs[it].z, hs[it].w};
        float y = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float abar = exp2_near_one_exact(delta * (a[i] * kLog2e));
            h[i] = fmaf(abar, h[i], dx * Bv[i]);
            y = fmaf(Cv[i], h[i], y);
        }
        y += __shfl_xor_sync(0xffffffffu, y, 1);
        y += __shfl_xor_sync(0xffffffffu, y, 2);
        if (live[it]) {
            __stcs(reinterpret_cast<float4*>(p.state + c * 16) + q, make_float4(h[0], h[1], h[2], h[3]));
            if (q == 0) {
                if (p.D != nullptr) y = fmaf(p.D[d], x, y);
                if (kHasZ) y *= silu_f32(load_as_float<IoT>(p.z, c));
                DType<IoT>::store(static_cast<IoT*>(p.out) + c, y);
            }
        }
    }
    }
}

template <typename IoT, typename BcT, bool kHasZ>
__global__ void __launch_bounds__(kUpdateThreads)
    state_update_generic_kernel(const __grid_constant__ UpdateParams p) {
    const int64_t chain = (int64_t)blockIdx.x * kUpdateThreads + threadIdx.x;
    if (chain >= p.chains) return;
    const int64_t b = chain / p.dim;
    const int64_t d = chain % p.dim;
    const float x = load_as_float<IoT>(p.x, chain);
    float s = load_as_float<IoT>(p.dt, chain);
    if (p.dt_bias != nullptr) s += p.dt_bias[d];
    const float delta = p.dt_softplus ? softplus_f32(s) : s;
    const float dx = delta * x;
    float y = 0.0f;
    for (int n = 0; n < p.dstate; ++n) {
        const float abar = exp2_near_one_exact(delta * (p.A[d * p.dstate + n] * kLog2e));
        float* hp = p.state + chain * p.dstate + n;
        const float h = fmaf(abar, *hp, dx * load_as_float<BcT>(p.B, b * p.dstate + n));
        *hp = h;
        y = fmaf(load_as_float<BcT>(p.C, b * p.dstate + n), h, y);
    }
    if (p.D != nullptr) y = fmaf(p.D[d], x, y);
    if (kHasZ) y *= silu_f32(load_as_float<IoT>(p.z, chain));
    DType<IoT>::store(static_cast<IoT*>(p.out) + chain, y);
}

}  // namespace mamba
