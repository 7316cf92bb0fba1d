// Short causal convolution of the Mamba block (sm_100a).
//
// Each channel d filters its inputs with W <= 4 taps over the most recent
// inputs ("Mamba 与状态空间模型", section 固定大小的状态: besides its 16 state
// numbers, each channel keeps a short convolution over its 4 most recent
// inputs):
//
//   out_t = act(bias_d + sum_{k<W} w_d,k x_{t-W+1+k}),   act = silu or identity,
//
// where x at negative times comes from a conv state holding the W most recent
// inputs, oldest first (zero without one).  The decode step shifts the state by
// one, appends x_t and applies the same sum.
//
// Both are HBM-bound streams: the prefill reads x and writes out once (the
// window's W-1 earlier elements come from the neighbouring lane by shuffle),
// the update reads and writes the 4-entry state of each chain.  Each thread
// carries several 16-byte loads (4 vectors, or 4 chains) to keep enough bytes
// in flight.
#pragma once

#include "ssm_device.cuh"

namespace mamba {

constexpr int kConvMaxWidth = MAMBA_MAX_CONV_WIDTH;
constexpr int kConvThreads = 256;

struct ConvParams {
    const void* x;
    const float* weight;       // (dim, W)
    const float* bias;         // (dim) or null
    const void* init;          // (batch, dim, W) or null
    void* out;
    void* final_state;         // (batch, dim, W) or null
    void* state;               // update: (batch, dim, W), in place
    int64_t batch, dim, seqlen, chains;
    int64_t vec_per_row;       // prefill vector path: 16-byte vectors per row
    int width;
    int silu;
};

template <typename IoT>
__device__ __forceinline__ float conv_load(const void* base, int64_t i) {
    return DType<IoT>::load(static_cast<const IoT*>(base) + i);
}

// Input x_s of chain `chain` for s < 0: the initial conv state (index W + s),
// or zero.
template <typename IoT>
__device__ __forceinline__ float conv_before_start(const ConvParams& p, int64_t chain, int64_t s) {
    return p.init != nullptr ? conv_load<IoT>(p.init, chain * p.width + (p.width + s)) : 0.0f;
}

__device__ __forceinline__ float conv_act(float acc, int silu) {
    return silu ? silu_f32(acc) : acc;
}

// Prefill, vector path (each row's start 16-byte aligned).  A warp covers
// kConvVecs x 32 consecutive 16-byte vectors of one row; lane l owns vectors
// base + 32 r + l (r < kConvVecs), each V consecutive time steps, and loads
// them all before computing, so every lane keeps kConvVecs loads in flight.
// The W-1 inputs before a vector are the last elements of the vector before it:
// lane l-1's (shuffle), lane 31's of the previous r for lane 0, or, for the
// warp's first vector, memory or the initial state at t = 0.
constexpr int kConvVecs = 4;

template <typename IoT, int kW>
__global__ void __launch_bounds__(kConvThreads)
    causal_conv1d_vec_kernel(const __grid_constant__ ConvParams p) {
    constexpr int V = 16 / (int)sizeof(IoT);
    constexpr int H = kW > 1 ? kW - 1 : 1;
    const int lane = threadIdx.x & 31;
    const int64_t warp_global = ((int64_t)blockIdx.x * kConvThreads + threadIdx.x) >> 5;
    const int64_t per_warp = 32 * kConvVecs;
    const int64_t blocks_per_row = (p.vec_per_row + per_warp - 1) / per_warp;
    const int64_t chain = warp_global / blocks_per_row;
    if (chain >= p.chains) return;                       // whole warp leaves together
    const int64_t base = (warp_global % blocks_per_row) * per_warp;
    const int64_t d = chain % p.dim;
    const IoT* row = static_cast<const IoT*>(p.x) + chain * p.seqlen;
    IoT* orow = static_cast<IoT*>(p.out) + chain * p.seqlen;

    uint4 raw[kConvVecs];
#pragma unroll
    for (int r = 0; r < kConvVecs; ++r) {
        const int64_t v = base + 32 * r + lane;
        raw[r] = v < p.vec_per_row ? *reinterpret_cast<const uint4*>(row + v * V)
                                   : make_uint4(0, 0, 0, 0);
    }
    float w[kW];
#pragma unroll
    for (int k = 0; k < kW; ++k) w[k] = p.weight[d * kW + k];
    const float b = p.bias != nullptr ? p.bias[d] : 0.0f;
    float prev_tail[H];                                  // lane's last H inputs of vector r-1
#pragma unroll
    for (int r = 0; r < kConvVecs; ++r) {
        const int64_t v = base + 32 * r + lane;
        const int64_t t0 = v * V;
        float xv[V];
        unpack16(raw[r], xv);
        float halo[H];
#pragma unroll
        for (int i = 0; i < kW - 1; ++i) {
            const float up = __shfl_up_sync(0xffffffffu, xv[V - (kW - 1) + i], 1);
            const float wrap = __shfl_sync(0xffffffffu, prev_tail[i], 31);
            float h = up;
            if (lane == 0) {
                const int64_t s = t0 - (kW - 1) + i;
                if (r > 0) h = wrap;
                else h = s >= 0 ? DType<IoT>::load(row + s) : conv_before_start<IoT>(p, chain, s);
            }
            halo[i] = h;
        }
#pragma unroll
        for (int i = 0; i < kW - 1; ++i) prev_tail[i] = xv[V - (kW - 1) + i];
        if (v < p.vec_per_row) {
            float o[V];
#pragma unroll
            for (int i = 0; i < V; ++i) {
                float acc = b;
#pragma unroll
                for (int k = 0; k < kW; ++k) {
                    const int j = i - (kW - 1) + k;     // element of this vector, or halo
                    acc = fmaf(w[k], j >= 0 ? xv[j] : halo[kW - 1 + j], acc);
                }
                o[i] = conv_act(acc, p.silu);
            }
            *reinterpret_cast<uint4*>(orow + t0) = pack16(o);
        }
    }
}

// Prefill, any alignment and length: one thread per output element.
template <typename IoT>
__global__ void __launch_bounds__(kConvThreads)
    causal_conv1d_generic_kernel(const __grid_constant__ ConvParams p) {
    const int64_t i = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
    if (i >= p.chains * p.seqlen) return;
    const int64_t chain = i / p.seqlen;
    const int64_t t = i % p.seqlen;
    const int64_t d = chain % p.dim;
    float acc = p.bias != nullptr ? p.bias[d] : 0.0f;
    for (int k = 0; k < p.width; ++k) {
        const int64_t s = t - (p.width - 1) + k;
        const float xs = s >= 0 ? conv_load<IoT>(p.x, chain * p.seqlen + s)
                                : conv_before_start<IoT>(p, chain, s);
        acc = fmaf(p.weight[d * p.width + k], xs, acc);
    }
    DType<IoT>::store(static_cast<IoT*>(p.out) + i, conv_act(acc, p.silu));
}

// Final conv state of the prefill: the last W inputs of (initial state ++ x).
// Index j reads position L - W + j >= j, so the initial state may be the
// final-state buffer itself.
template <typename IoT>
__global__ void __launch_bounds__(kConvThreads)
    causal_conv1d_final_state_kernel(const __grid_constant__ ConvParams p) {
    const int64_t chain = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
    if (chain >= p.chains) return;
    IoT* fs = static_cast<IoT*>(p.final_state) + chain * p.width;
    for (int j = 0; j < p.width; ++j) {
        const int64_t s = p.seqlen - p.width + j;
        const float v = s >= 0 ? conv_load<IoT>(p.x, chain * p.seqlen + s)
                               : conv_before_start<IoT>(p, chain, s);
        DType<IoT>::store(fs + j, v);
    }
}

// Decode: one thread per chain; the W-entry state is shifted in place.
template <typename IoT>
__global__ void __launch_bounds__(kConvThreads)
    causal_conv1d_update_kernel(const __grid_constant__ ConvParams p) {
    const int64_t chain = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
    if (chain >= p.chains) return;
    const int64_t d = chain % p.dim;
    IoT* st = static_cast<IoT*>(p.state) + chain * p.width;
    const float xin = conv_load<IoT>(p.x, chain);
    float cur[kConvMaxWidth];
#pragma unroll
    for (int j = 0; j < kConvMaxWidth; ++j)   // old state entries 1..W-1, then x
        cur[j] = j + 1 < p.width ? DType<IoT>::load(st + j + 1) : (j + 1 == p.width ? xin : 0.0f);
    float acc = p.bias != nullptr ? p.bias[d] : 0.0f;
#pragma unroll
    for (int k = 0; k < kConvMaxWidth; ++k)
        if (k < p.width) {
            acc = fmaf(p.weight[d * p.width + k], cur[k], acc);
            DType<IoT>::store(st + k, cur[k]);
        }
    DType<IoT>::store(static_cast<IoT*>(p.out) + chain, conv_act(acc, p.silu));
}

// Decode, W = 4 with the state 8- (bf16) or 16-byte (fp32) aligned: the
// state moves as one vector each way.
template <typename IoT>
__global__ void __launch_bounds__(kConvThreads)
    causal_conv1d_update_w4_kernel(const __grid_constant__ ConvParams p) {
    const int64_t chain = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
    if (chain >= p.chains) return;
    const int64_t d = chain % p.dim;
    float cur[4];
    if constexpr (sizeof(IoT) == 2) {
        uint2* sp = reinterpret_cast<uint2*>(static_cast<IoT*>(p.state) + chain * 4);
        const uint2 s = *sp;
        cur[0] = __uint_as_float(s.x & 0xffff0000u);            // old[1]
        cur[1] = __uint_as_float(s.y << 16);                     // old[2]
        cur[2] = __uint_as_float(s.y & 0xffff0000u);            // old[3]
        cur[3] = conv_load<IoT>(p.x, chain);
        *sp = make_uint2(pack_bf16x2(cur[0], cur[1]), pack_bf16x2(cur[2], cur[3]));
    } else {
        float4* sp = reinterpret_cast<float4*>(static_cast<IoT*>(p.state) + chain * 4);
        const float4 s = *sp;
        cur[0] = s.y;
        cur[1] = s.z;
        cur[2] = s.w;
        cur[3] = conv_load<IoT>(p.x, chain);
        *sp = make_float4(cur[0], cur[1], cur[2], cur[3]);
    }
    const float4 w = *reinterpret_cast<const float4*>(p.weight + d * 4);
    float acc = p.bias != nullptr ? p.bias[d] : 0.0f;
    acc = fmaf(w.x, cur[0], acc);
    acc = fmaf(w.y, cur[1], acc);
    acc = fmaf(w.z, cur[2], acc);
    acc = fmaf(w.w, cur[3], acc);
    DType<IoT>::store(static_cast<IoT*>(p.out) + chain, conv_act(acc, p.silu));
}

// Decode, W = 4, kC chains per thread (kC = 2 or 4): the kC 4-entry states
// (8 kC bytes in bf16, 16 kC in fp32), the inputs and the outputs move as
// vectors.  Needs the state aligned to its vector and x/out to kC elements;
// the last chains (a count not a multiple of kC) go one by one.
template <typename IoT>
__device__ __forceinline__ float conv4_sum(const ConvParams& p, int64_t chain, const float (&cur)[4]) {
    const float4 w = *reinterpret_cast<const float4*>(p.weight + (chain % p.dim) * 4);
    float acc = p.bias != nullptr ? p.bias[chain % p.dim] : 0.0f;
    acc = fmaf(w.x, cur[0], acc);
    acc = fmaf(w.y, cur[1], acc);
    acc = fmaf(w.z, cur[2], acc);
    acc = fmaf(w.w, cur[3], acc);
    return conv_act(acc, p.silu);
}

// kC consecutive elements of type IoT as fp32, and back (one vector access).
template <typename IoT, int kC>
__device__ __forceinline__ void load_vec(const IoT* src, float (&v)[kC]) {
    static_assert(kC * sizeof(IoT) == 4 || kC * sizeof(IoT) == 8 || kC * sizeof(IoT) == 16, "vector");
    if constexpr (sizeof(IoT) == 2) {
        uint32_t w[kC / 2];
        if constexpr (kC == 2) w[0] = *reinterpret_cast<const uint32_t*>(src);
        else { const uint2 t = *reinterpret_cast<const uint2*>(src); w[0] = t.x; w[1] = t.y; }
#pragma unroll
        for (int i = 0; i < kC / 2; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
        if constexpr (kC == 2) { const float2 t = *reinterpret_cast<const float2*>(src); v[0] = t.x; v[1] = t.y; }
        else { const float4 t = *reinterpret_cast<const float4*>(src); v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w; }
    }
}

template <typename IoT, int kC>
__device__ __forceinline__ void store_vec(IoT* dst, const float (&v)[kC]) {
    if constexpr (sizeof(IoT) == 2) {
        if constexpr (kC == 2) *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(v[0], v[1]);
        else *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    } else {
        if constexpr (kC == 2) *reinterpret_cast<float2*>(dst) = make_float2(v[0], v[1]);
        else *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
    }
}

// kPdl: launched as a programmatic dependent launch.  The next launch on the
// stream may start at once; this one reads its own conv state, then waits for
// the previous launch to complete before it reads x and writes anything (the
// caller guarantees that the previous launch neither reads nor writes this
// call's state).
template <typename IoT, int kC, bool kPdl>
__global__ void __launch_bounds__(kConvThreads)
    causal_conv1d_update_w4xn_kernel(const __grid_constant__ ConvParams p) {
    if (kPdl) grid_launch_dependents();
    const int64_t c0 = kC * ((int64_t)blockIdx.x * kConvThreads + threadIdx.x);
    if (c0 >= p.chains) {
        if (kPdl) grid_dependency_wait();
        return;
    }
    IoT* st = static_cast<IoT*>(p.state) + c0 * 4;
    const IoT* xs = static_cast<const IoT*>(p.x) + c0;
    IoT* os = static_cast<IoT*>(p.out) + c0;
    if (c0 + kC > p.chains) {                           // tail, one chain at a time
        if (kPdl) grid_dependency_wait();
        for (int64_t c = c0; c < p.chains; ++c) {
            IoT* sc = st + (c - c0) * 4;
            const float cur[4] = {DType<IoT>::load(sc + 1), DType<IoT>::load(sc + 2),
                                  DType<IoT>::load(sc + 3), DType<IoT>::load(xs + (c - c0))};
            for (int j = 0; j < 4; ++j) DType<IoT>::store(sc + j, cur[j]);
            DType<IoT>::store(os + (c - c0), conv4_sum<IoT>(p, c, cur));
        }
        return;
    }
    float old[4 * kC], xin[kC];
#pragma unroll
    for (int c = 0; c < kC; ++c) {
        float v[4];
        load_vec<IoT, 4>(st + 4 * c, v);
#pragma unroll
        for (int j = 0; j < 4; ++j) old[4 * c + j] = v[j];
    }
    if (kPdl) grid_dependency_wait();
    load_vec<IoT, kC>(xs, xin);
    float o[kC];
#pragma unroll
    for (int c = 0; c < kC; ++c) {
        const float cur[4] = {old[4 * c + 1], old[4 * c + 2], old[4 * c + 3], xin[c]};
        store_vec<IoT, 4>(st + 4 * c, cur);
        o[c] = conv4_sum<IoT>(p, c0 + c, cur);
    }
    store_vec<IoT, kC>(os, o);
}

#ifndef MAMBA_CONV_UPDATE_CHAINS
#define MAMBA_CONV_UPDATE_CHAINS 2
#endif
constexpr int kConvUpdateChains = MAMBA_CONV_UPDATE_CHAINS;   // chains per thread (W = 4)

}  // namespace mamba
