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
// memory-bound kernel has ALU time to spare.  With MAMBA_FLAG_ZOH every path
// multiplies the input term by the zero-order-hold gain zoh_phi ("超越注意力：
// 探索Mamba与状态空间模型", section 状态空间模型基础).
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
    int zoh;             // zero-order-hold input term Delta phi(Delta A) B x
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
            const float x2 = delta * (a[i] * kLog2e);
            const float abar = exp2_near_one_exact(x2);
            const float gx = p.zoh ? dx * zoh_phi(x2, abar) : dx;
            h[i] = fmaf(abar, h[i], gx * Bv[i]);
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

// ----------------------------------------------------------------------------
// Streaming path (N = 16, dim % 8 == 0, 16-byte aligned buffers).
//
// Each CTA owns one block of kBulkTile channels and walks batch rows; the
// block's A rows, D and dt_bias stay in registers.  A producer warp keeps a
// kBulkStages-deep ring of tiles loading by 1-D bulk TMA (the tile's fp32
// state, x, dt, z and the batch row's B and C).  Four consumer warps each own
// 32 channels of the tile: they update the state in place in shared memory,
// write the outputs beside it, bulk-store their slice back, and release the
// stage through an mbarrier once the store has read it.  No CTA-wide barrier
// sits on the path, so the ring keeps several tiles in flight per CTA.  Four
// lanes share a chain (a float4 of state each); softplus and silu run once per
// chain, spread over the four lanes, and are exchanged by shuffles.  Abar is
// MUFU ex2 for bf16 inputs and exp2_near_one_exact for fp32 inputs, as in the
// scan.  kZoh, the zero-order-hold gain zoh_phi, is a separate instance (4
// CTAs per SM) so that the Euler one keeps 5 CTAs per SM.
// kPdl is the instance for a programmatic dependent launch (MAMBA_FLAG_PDL):
// the grid may start while the previous kernel on the stream finishes, so the
// producer first requests the state of its first tiles, then waits for that
// kernel before the token inputs, and lets the next launch start once its last
// loads are issued.  That instance runs 4 CTAs per SM, which leaves room for
// the next launch's CTAs to start early; the plain instance runs 5.
constexpr int kBulkConsumers = 4;
constexpr int kBulkThreads = 32 * (kBulkConsumers + 1);
constexpr int kBulkTile = 32 * kBulkConsumers;       // channels per tile
constexpr int kBulkStages = 4;
constexpr int kBOffState = 0;                        // kBulkTile x 64 B
constexpr int kBOffX = kBulkTile * 64;               // kBulkTile x up to 4 B each:
constexpr int kBOffDt = kBOffX + kBulkTile * 4;
constexpr int kBOffZ = kBOffDt + kBulkTile * 4;
constexpr int kBOffOut = kBOffZ + kBulkTile * 4;
constexpr int kBOffB = kBOffOut + kBulkTile * 4;     // 16 x up to 4 B
constexpr int kBOffC = kBOffB + 64;
constexpr int kBStage = ((kBOffC + 64 + 127) / 128) * 128;
constexpr int kBulkSmemBytes = kBulkStages * kBStage + 2 * kBulkStages * 8 + 1024;

template <typename IoT, typename BcT, bool kHasZ, bool kZoh, bool kPdl>
__global__ void __launch_bounds__(kBulkThreads)
    state_update_bulk_kernel(const __grid_constant__ UpdateParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBulkStages * kBStage);
    uint64_t* empty = full + kBulkStages;
    constexpr int ES = (int)sizeof(IoT);
    constexpr int BS = (int)sizeof(BcT);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // This CTA: channel block `blk`, batch rows b0, b0 + bstep, ...
    const int nblk = (int)((p.dim + kBulkTile - 1) / kBulkTile);
    const int blk = (int)(blockIdx.x % nblk);
    const int64_t b0 = blockIdx.x / nblk;
    const int64_t bstep = max(1u, gridDim.x / (unsigned)nblk);
    const int64_t d0 = (int64_t)blk * kBulkTile;
    const int nch = (int)min((int64_t)kBulkTile, p.dim - d0);
    const int64_t mine = b0 < p.batch ? (p.batch - b0 + bstep - 1) / bstep : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kBulkStages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), kBulkConsumers);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kBulkConsumers) {
        // ---------------- producer ----------------
        if (lane != 0) return;
        const uint32_t tok = (uint32_t)nch * ES;
        const uint32_t bytes = (uint32_t)nch * 64 + (kHasZ ? 3u : 2u) * tok + 2u * 16u * BS;
        auto load_state = [&](int64_t k) {
            const int s = (int)(k % kBulkStages);
            const int64_t c0 = (b0 + k * bstep) * p.dim + d0;
            const uint32_t bar = smem_u32(&full[s]);
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(bar, bytes);
            bulk_load(smem_u32(smem + s * kBStage + kBOffState), p.state + c0 * 16, (uint32_t)nch * 64, bar);
        };
        auto load_tokens = [&](int64_t k) {
            const int s = (int)(k % kBulkStages);
            const int64_t b = b0 + k * bstep;
            const int64_t c0 = b * p.dim + d0;
            uint8_t* st = smem + s * kBStage;
            const uint32_t bar = smem_u32(&full[s]);
            bulk_load(smem_u32(st + kBOffX), static_cast<const IoT*>(p.x) + c0, tok, bar);
            bulk_load(smem_u32(st + kBOffDt), static_cast<const IoT*>(p.dt) + c0, tok, bar);
            if (kHasZ) bulk_load(smem_u32(st + kBOffZ), static_cast<const IoT*>(p.z) + c0, tok, bar);
            bulk_load(smem_u32(st + kBOffB), static_cast<const BcT*>(p.B) + b * 16, 16 * BS, bar);
            bulk_load(smem_u32(st + kBOffC), static_cast<const BcT*>(p.C) + b * 16, 16 * BS, bar);
        };
        // The state belongs to this call alone, so the first tiles' state is
        // requested before waiting for the kernel this one may overlap with
        // (programmatic dependent launch); the token inputs may come from it.
        const int64_t pre = kPdl ? (mine < kBulkStages ? mine : kBulkStages) : 0;
        if constexpr (kPdl) {
            for (int64_t k = 0; k < pre; ++k) load_state(k);
            grid_dependency_wait();
            for (int64_t k = 0; k < pre; ++k) load_tokens(k);
        }
        int64_t k = pre;
        for (; k < mine; ++k) {
            const int s = (int)(k % kBulkStages);
            if (k >= kBulkStages &&
                !mbar_wait_bounded(smem_u32(&empty[s]), (uint32_t)((k / kBulkStages - 1) & 1))) {
                record_device_error(MAMBA_ERR_TIMEOUT);
                break;
            }
            load_state(k);
            load_tokens(k);
        }
        if constexpr (kPdl) grid_launch_dependents();
        // Loads still in flight must land before the CTA's shared memory goes away.
        for (int64_t j = max((int64_t)0, k - kBulkStages); j < k; ++j)
            (void)mbar_wait_bounded(smem_u32(&full[j % kBulkStages]), (uint32_t)((j / kBulkStages) & 1));
        return;
    }

    // ---------------- consumers ----------------
    // Lane l of warp w holds quarter q = l & 3 of chain 32 w + 8 it + (l >> 2)
    // for items it = 0..3.  The four lanes of a quad also split the per-chain
    // scalar work: lane q computes softplus and silu for item q.
    constexpr bool kExact = sizeof(IoT) == 4;
    const int q = lane & 3;
    const int quad = lane & ~3;
    constexpr int kItems = 4;
    float2 a01[kItems], a23[kItems];
    int ch[kItems];
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        ch[it] = 32 * warp + 8 * it + (lane >> 2);
        const int64_t d = d0 + (ch[it] < nch ? ch[it] : 0);
        const float4 av = *(reinterpret_cast<const float4*>(p.A + d * 16) + q);
        a01[it] = __fmul2_rn(make_float2(av.x, av.y), make_float2(kLog2e, kLog2e));
        a23[it] = __fmul2_rn(make_float2(av.z, av.w), make_float2(kLog2e, kLog2e));
    }
    // Per-chain parameters of item q (this lane's scalar duty).
    const int my_ch = 32 * warp + 8 * q + (lane >> 2);   // chain of item q
    const bool my_live = my_ch < nch;
    const int64_t my_d = d0 + (my_live ? my_ch : 0);
    const float my_D = p.D != nullptr ? p.D[my_d] : 0.0f;
    const float my_bias = p.dt_bias != nullptr ? p.dt_bias[my_d] : 0.0f;
    const int nw = max(0, min(32, nch - 32 * warp));   // this warp's chains in a tile

    for (int64_t k = 0; k < mine; ++k) {
        const int s = (int)(k % kBulkStages);
        uint8_t* st = smem + s * kBStage;
        bool ok = mbar_wait_bounded(smem_u32(&full[s]), (uint32_t)((k / kBulkStages) & 1));
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
            if (lane == 0) record_device_error(MAMBA_ERR_TIMEOUT);
            break;
        }
        const IoT* xs = reinterpret_cast<const IoT*>(st + kBOffX);
        const BcT* Bs = reinterpret_cast<const BcT*>(st + kBOffB) + 4 * q;
        const BcT* Cs = reinterpret_cast<const BcT*>(st + kBOffC) + 4 * q;
        const float2 b01 = make_float2(DType<BcT>::load(Bs), DType<BcT>::load(Bs + 1));
        const float2 b23 = make_float2(DType<BcT>::load(Bs + 2), DType<BcT>::load(Bs + 3));
        const float2 c01 = make_float2(DType<BcT>::load(Cs), DType<BcT>::load(Cs + 1));
        const float2 c23 = make_float2(DType<BcT>::load(Cs + 2), DType<BcT>::load(Cs + 3));
        // Delta of item q's chain, computed by this lane.
        const int mc = my_live ? my_ch : 0;
        const float my_s = DType<IoT>::load(reinterpret_cast<const IoT*>(st + kBOffDt) + mc) + my_bias;
        const float my_delta = p.dt_softplus ? softplus_f32(my_s) : my_s;
        float y_item[kItems];
#pragma unroll
        for (int it = 0; it < kItems; ++it) {
            const int c = ch[it] < nch ? ch[it] : 0;
            const float4 hs = reinterpret_cast<const float4*>(st + kBOffState)[4 * c + q];
            const float x = DType<IoT>::load(xs + c);
            const float delta = __shfl_sync(0xffffffffu, my_delta, quad | it);
            const float dx = delta * x;
            const float2 d2 = make_float2(delta, delta);
            const float2 dx2 = make_float2(dx, dx);
            const float2 x01 = __fmul2_rn(d2, a01[it]);
            const float2 x23 = __fmul2_rn(d2, a23[it]);
            const float2 e01 = kExact ? exp2_near_one_exact2(x01)
                                      : make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
            const float2 e23 = kExact ? exp2_near_one_exact2(x23)
                                      : make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
            float2 in01 = __fmul2_rn(dx2, b01);
            float2 in23 = __fmul2_rn(dx2, b23);
            if (kZoh) {
                in01 = __fmul2_rn(in01, make_float2(zoh_phi(x01.x, e01.x), zoh_phi(x01.y, e01.y)));
                in23 = __fmul2_rn(in23, make_float2(zoh_phi(x23.x, e23.x), zoh_phi(x23.y, e23.y)));
            }
            const float2 h01 = __ffma2_rn(e01, make_float2(hs.x, hs.y), in01);
            const float2 h23 = __ffma2_rn(e23, make_float2(hs.z, hs.w), in23);
            const float2 yy = __ffma2_rn(c23, h23, __fmul2_rn(c01, h01));
            float y = yy.x + yy.y;
            y += __shfl_xor_sync(0xffffffffu, y, 1);
            y += __shfl_xor_sync(0xffffffffu, y, 2);
            y_item[it] = y;
            if (ch[it] < nch)
                reinterpret_cast<float4*>(st + kBOffState)[4 * c + q] =
                    make_float4(h01.x, h01.y, h23.x, h23.y);
        }
        // Output of item q's chain, by this lane.
        float y = y_item[0];
#pragma unroll
        for (int it = 1; it < kItems; ++it)
            if (q == it) y = y_item[it];
        if (my_live) {
            y = fmaf(my_D, DType<IoT>::load(xs + my_ch), y);
            if (kHasZ) y *= silu_f32(DType<IoT>::load(reinterpret_cast<const IoT*>(st + kBOffZ) + my_ch));
            DType<IoT>::store(reinterpret_cast<IoT*>(st + kBOffOut) + my_ch, y);
        }
        // Store this warp's slice, then hand the stage back to the producer.
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            if (nw > 0) {
                const int64_t c0 = (b0 + k * bstep) * p.dim + d0 + 32 * warp;
                bulk_store(p.state + c0 * 16, smem_u32(st + kBOffState + 32 * warp * 64),
                           (uint32_t)nw * 64);
                bulk_store(static_cast<IoT*>(p.out) + c0, smem_u32(st + kBOffOut + 32 * warp * ES),
                           (uint32_t)nw * ES);
                bulk_commit();
                bulk_wait_read<0>();
            }
            mbar_arrive(smem_u32(&empty[s]));
        }
    }
    if (lane == 0) bulk_wait<0>();
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
        const float x2 = delta * (p.A[d * p.dstate + n] * kLog2e);
        const float abar = exp2_near_one_exact(x2);
        const float gx = p.zoh ? dx * zoh_phi(x2, abar) : dx;
        float* hp = p.state + chain * p.dstate + n;
        const float h = fmaf(abar, *hp, gx * load_as_float<BcT>(p.B, b * p.dstate + n));
        *hp = h;
        y = fmaf(load_as_float<BcT>(p.C, b * p.dstate + n), h, y);
    }
    if (p.D != nullptr) y = fmaf(p.D[d], x, y);
    if (kHasZ) y *= silu_f32(load_as_float<IoT>(p.z, chain));
    DType<IoT>::store(static_cast<IoT*>(p.out) + chain, y);
}

}  // namespace mamba
