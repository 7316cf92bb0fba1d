// Carry and correction passes of the scan's parallel mode (sm_100a).
//
// The parallel mode runs every segment k of a sequence at once from a zero
// start (segment 0 from the given start state).  Each segment leaves, per
// chain and state entry n, its end state e0_k,n and its sum of Delta s_k.
// Over a segment the recurrence h_t = Abar_t h_{t-1} + b_t is affine in the
// state it starts from: starting from h_in instead of zero adds
// P_t,n h_in,n with P_t,n = prod_{r<=t} Abar_r,n = exp(A_n S_t), S_t the sum of
// Delta over the segment's steps up to t.  Hence:
//
//  * scan_carry_kernel: the true end states follow the associative combine of
//    the parallel scan, (P1, h1) then (P2, h2) -> (P1 P2, P2 h1 + h2)
//    ("Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
//    section 硬件效率), over the pairs (exp(A_n s_k), e0_k,n).  One warp per
//    chain scans 32 segments at a time with warp shuffles and carries the
//    running state from one group of 32 to the next.  The inclusive results
//    overwrite the end states in place: slot k - 1 becomes segment k's start
//    state, and the last slot the chain's last_state.
//
//  * scan_correct_kernel: segment k >= 1 then adds to each output
//    y_t += C_t . (P_t (.) h_in), times silu(z_t) when gated.  The term has no
//    recurrence, so one warp walks a segment with its lanes over consecutive
//    time steps: Delta, its running sum S_t (warp-shuffle prefix sum), 16
//    exponentials and a dot product per step.  Where Delta >= 0 throughout
//    (softplus on) S_t never decreases, so once A_n S_t < -127 the term of
//    state entry n is below 2^-127 for the rest of the segment, which
//    ex2.approx.ftz returns as 0: the entry drops out of the walk, and the walk
//    stops when none is left.  The outputs are exactly those of walking on to
//    the segment's end, which is where a segment with slow decay stops anyway.
#pragma once

#include "ssm_device.cuh"

namespace mamba {

constexpr int kCarryWarps = 4;        // warps (chains) per CTA of the carry pass
constexpr int kCorrectWarps = 8;      // warps per CTA of the correction pass
constexpr float kUnderflowLog2 = -127.0f;

struct CarryParams {
    const float* A;          // (dim, dstate)
    float* ws_h;             // [K][chains][16]: end states from each segment's own start; in place
    const float* ws_sdt;     // [K][chains]: sum of Delta per segment
    float* last_state;       // (batch, dim, dstate) or null
    int64_t chains, dim;
    int nseg, dstate;
};

// One warp per chain; lane l holds segments k0 + l of the current group of 32.
template <bool kExact>
__global__ void __launch_bounds__(kCarryWarps * 32)
    scan_carry_kernel(const __grid_constant__ CarryParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t chain = (int64_t)blockIdx.x * kCarryWarps + warp;
    if (chain >= p.chains) return;
    const int64_t d = chain % p.dim;
    for (int n = 0; n < p.dstate; ++n) {
        const float a2 = p.A[d * p.dstate + n] * kLog2e;
        float carry = 0.0f;   // true end state of the segment before this group
        for (int k0 = 0; k0 < p.nseg; k0 += 32) {
            const int k = k0 + lane;
            float P = 1.0f, h = 0.0f;   // the identity pair beyond the last segment
            float* slot = p.ws_h + ((int64_t)k * p.chains + chain) * kNPad + n;
            if (k < p.nseg) {
                h = __ldcg(slot);
                const float x = a2 * __ldcg(p.ws_sdt + (int64_t)k * p.chains + chain);
                P = kExact ? exp2_near_one_exact(x) : ex2_approx(x);
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {   // inclusive scan; the lower lane is earlier
                const float Pe = __shfl_up_sync(0xffffffffu, P, o);
                const float he = __shfl_up_sync(0xffffffffu, h, o);
                if (lane >= o) {
                    h = fmaf(P, he, h);
                    P *= Pe;
                }
            }
            const float e = fmaf(P, carry, h);
            if (k < p.nseg) __stcg(slot, e);
            carry = __shfl_sync(0xffffffffu, e, 31);
        }
        if (lane == 0 && p.last_state != nullptr) p.last_state[chain * p.dstate + n] = carry;
    }
}

struct CorrectParams {
    const void* delta;       // (batch, dim, L)
    const void* z;           // (batch, dim, L) or null
    const void* C;           // (batch, dstate, L)
    const float* A;          // (dim, dstate)
    const float* delta_bias; // (dim) or null
    void* out;               // (batch, dim, L), corrected in place
    const float* ws_h;       // [K][chains][16]: slot k - 1 = start state of segment k
    unsigned int* counter;   // dequeue counter
    int64_t batch, dim, seqlen, chains, seg_len, items;
    int nseg, dstate;
    int bc_bf16;
    int vec_io;              // 16-byte loads and stores of delta, z, out rows are aligned
    int vec_c;               // 16-byte loads of C rows are aligned
};

// V consecutive values of a row starting at element `t` as fp32: one or two
// 16-byte loads when `vec`, else element by element (0 past `valid`).
template <typename T, int V>
__device__ __forceinline__ void load_run(const T* row, int64_t t, int valid, bool vec, float (&f)[V]) {
    constexpr bool kWhole = (V * sizeof(T)) % 16 == 0;   // V values fill whole 16-byte vectors
    if (kWhole && vec && valid == V) {
        constexpr int per = 16 / (int)sizeof(T);
#pragma unroll
        for (int q = 0; q < V / per; ++q) {
            const uint4 v = __ldcs(reinterpret_cast<const uint4*>(row + t) + q);
            if (sizeof(T) == 2) {
                float g[8];
                unpack16(v, g);
#pragma unroll
                for (int j = 0; j < per; ++j) f[q * per + j] = g[j];
            } else {
                float g[4];
                unpack16(v, g);
#pragma unroll
                for (int j = 0; j < per; ++j) f[q * per + j] = g[j];
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < V; ++j) f[j] = j < valid ? DType<T>::load(row + t + j) : 0.0f;
    }
}

// The same V values, kept as raw words (V * size / 4 of them) so that a pass
// can have every load in flight before it uses any: one or two 16-byte loads
// when `vec`, else element by element (0 past `valid`).
template <typename T, int V>
struct RawRun {
    static constexpr int kWords = V * (int)sizeof(T) / 4;
    uint32_t w[kWords];
};

template <typename T, int V>
__device__ __forceinline__ void load_raw(const T* row, int64_t t, int valid, bool vec,
                                         RawRun<T, V>& r) {
    constexpr int kWords = RawRun<T, V>::kWords;
    if (kWords % 4 == 0 && vec && valid == V) {
#pragma unroll
        for (int q = 0; q < kWords / 4; ++q) {
            const uint4 v = __ldcs(reinterpret_cast<const uint4*>(row + t) + q);
            r.w[4 * q] = v.x; r.w[4 * q + 1] = v.y; r.w[4 * q + 2] = v.z; r.w[4 * q + 3] = v.w;
        }
    } else if constexpr (sizeof(T) == 2) {
        const unsigned short* h = reinterpret_cast<const unsigned short*>(row + t);
#pragma unroll
        for (int i = 0; i < kWords; ++i) {
            const uint32_t lo = 2 * i < valid ? h[2 * i] : 0u;
            const uint32_t hi = 2 * i + 1 < valid ? h[2 * i + 1] : 0u;
            r.w[i] = lo | (hi << 16);
        }
    } else {
        const uint32_t* f = reinterpret_cast<const uint32_t*>(row + t);
#pragma unroll
        for (int i = 0; i < kWords; ++i) r.w[i] = i < valid ? f[i] : 0u;
    }
}

// Value j of a raw run, as fp32.
template <typename T, int V>
__device__ __forceinline__ float raw_elem(const RawRun<T, V>& r, int j) {
    if constexpr (sizeof(T) == 2) {
        const uint32_t w = r.w[j >> 1];
        return __uint_as_float((j & 1) ? (w & 0xffff0000u) : (w << 16));
    } else {
        return __uint_as_float(r.w[j]);
    }
}

// Segment k's correction for one chain (one warp, lanes over time): adds
// C_t . (exp(A S_t) (.) hin) (gated) to the segment's outputs, hin being the
// segment's true start state.  Every lane holds the same hin.  With kAhead a
// pass issues all its loads (delta, out, z and the C rows of the live state
// entries) before it uses any, so their latencies overlap; without it (the
// look-back inside the scan kernel, short of registers) each C row is loaded
// where its entry is taken.
template <typename IoT, typename BcT, bool kHasZ, bool kSoftplus, bool kAhead = false>
__device__ __forceinline__ void correct_chain(const CorrectParams& p, int64_t chain, int64_t k,
                                              const float (&hin)[kNPad], int lane) {
    constexpr int V = 16 / (int)sizeof(IoT);    // steps per lane and pass
    constexpr bool kExact = sizeof(IoT) == 4;
    const IoT* delta = static_cast<const IoT*>(p.delta);
    const IoT* zz = static_cast<const IoT*>(p.z);
    const BcT* Cm = static_cast<const BcT*>(p.C);
    IoT* out = static_cast<IoT*>(p.out);
    const int64_t b = chain / p.dim, d = chain % p.dim;
    const int64_t t_begin = k * p.seg_len;
    const int64_t t_end = min(t_begin + p.seg_len, p.seqlen);
    float a2[kNPad];
#pragma unroll
    for (int n = 0; n < kNPad; ++n) a2[n] = n < p.dstate ? p.A[d * p.dstate + n] * kLog2e : 0.0f;
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.0f;
    const IoT* drow = delta + chain * p.seqlen;
    const IoT* zrow = kHasZ ? zz + chain * p.seqlen : nullptr;
    IoT* orow = out + chain * p.seqlen;
    const BcT* crow = Cm + b * p.dstate * p.seqlen;
    float S_run = 0.0f;       // sum of Delta before this pass's first step
    bool monotone = true;     // Delta >= 0 at every step so far

    for (int64_t t0 = t_begin; t0 < t_end; t0 += 32 * V) {
        // State entries whose exp(A_n S_t) is below 2^-127 for the rest of
        // the segment (0 after ex2.approx.ftz) drop out; none left, done.
        uint32_t active = 0;
#pragma unroll
        for (int n = 0; n < kNPad; ++n)
            if (n < p.dstate && !(monotone && a2[n] < 0.0f && a2[n] * S_run < kUnderflowLog2))
                active |= 1u << n;
        if (active == 0) break;
        const int64_t ts = t0 + (int64_t)lane * V;
        const int valid = (int)max((int64_t)0, min((int64_t)V, t_end - ts));
        RawRun<BcT, V> craw[kAhead ? kNPad : 1];
        RawRun<IoT, V> oraw, zraw;
        float dl[V];
        if constexpr (kAhead) {
            RawRun<IoT, V> draw;
            load_raw<IoT, V>(drow, ts, valid, p.vec_io != 0, draw);
#pragma unroll
            for (int n = 0; n < kNPad; ++n) {
                if ((active >> n) & 1u) {
                    load_raw<BcT, V>(crow + n * p.seqlen, ts, valid, p.vec_c != 0, craw[n]);
                } else {
#pragma unroll
                    for (int i = 0; i < RawRun<BcT, V>::kWords; ++i) craw[n].w[i] = 0u;
                }
            }
            load_raw<IoT, V>(orow, ts, valid, p.vec_io != 0, oraw);
            if (kHasZ) load_raw<IoT, V>(zrow, ts, valid, p.vec_io != 0, zraw);
#pragma unroll
            for (int j = 0; j < V; ++j) dl[j] = raw_elem<IoT, V>(draw, j);
        } else {
            load_run<IoT, V>(drow, ts, valid, p.vec_io != 0, dl);
        }
        float S[V];
        float run = 0.0f;
        bool nonneg = true;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            float dt = 0.0f;
            if (j < valid) {
                const float sarg = dl[j] + bias;
                dt = kSoftplus ? (kExact ? softplus_f32(sarg) : softplus_lg2(sarg)) : sarg;
            }
            nonneg = nonneg && dt >= 0.0f;
            run += dt;
            S[j] = run;
        }
        // exclusive prefix of the lanes' totals, then this pass's total
        float incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const float before = S_run + (incl - run);
        S_run += __shfl_sync(0xffffffffu, incl, 31);
        monotone = __all_sync(0xffffffffu, monotone && nonneg) != 0;
        if (valid == 0) continue;

        float corr[V];
#pragma unroll
        for (int j = 0; j < V; ++j) corr[j] = 0.0f;
#pragma unroll
        for (int n = 0; n < kNPad; ++n) {
            if (!((active >> n) & 1u)) continue;   // uniform across the warp
            float cv[V];
            if constexpr (kAhead) {
#pragma unroll
                for (int j = 0; j < V; ++j) cv[j] = raw_elem<BcT, V>(craw[n], j);
            } else {
                load_run<BcT, V>(crow + n * p.seqlen, ts, valid, p.vec_c != 0, cv);
            }
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const float x = a2[n] * (before + S[j]);
                corr[j] = fmaf(cv[j] * ex2_approx(x), hin[n], corr[j]);
            }
        }
        float o[V];
        float zv[V];
        if constexpr (kAhead) {
#pragma unroll
            for (int j = 0; j < V; ++j) {
                o[j] = raw_elem<IoT, V>(oraw, j);
                if (kHasZ) zv[j] = raw_elem<IoT, V>(zraw, j);
            }
        } else {
            load_run<IoT, V>(orow, ts, valid, p.vec_io != 0, o);
            if (kHasZ) load_run<IoT, V>(zrow, ts, valid, p.vec_io != 0, zv);
        }
#pragma unroll
        for (int j = 0; j < V; ++j) {
            float g = corr[j];
            if (kHasZ) g *= kExact ? silu_f32(zv[j]) : silu_tanh(zv[j]);
            o[j] += g;
        }
        if (p.vec_io != 0 && valid == V) {
            if (sizeof(IoT) == 2) {
                float f8[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) f8[j] = o[j];
                *reinterpret_cast<uint4*>(orow + ts) = pack16(f8);
            } else {
                float f4[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) f4[j] = o[j];
                *reinterpret_cast<uint4*>(orow + ts) = pack16(f4);
            }
        } else {
            for (int j = 0; j < valid; ++j) DType<IoT>::store(orow + ts + j, o[j]);
        }
    }
}

template <typename IoT, typename BcT, bool kHasZ, bool kSoftplus>
// Two CTAs (16 warps) per SM: the pass's loads all in flight take registers,
// and capping them at 128 keeps the 16 warps (measured faster than 8 warps at
// 168 registers).
__global__ void __launch_bounds__(kCorrectWarps * 32, 2)
    scan_correct_kernel(const __grid_constant__ CorrectParams p) {
    const int lane = threadIdx.x & 31;
    for (;;) {
        unsigned int item = 0;
        if (lane == 0) item = atomicAdd(p.counter, 1u);
        item = __shfl_sync(0xffffffffu, item, 0);
        if ((int64_t)item >= p.items) break;
        const int64_t chain = item % p.chains;
        const int64_t k = 1 + item / p.chains;
        float hin[kNPad];
        const float* hs = p.ws_h + ((k - 1) * p.chains + chain) * kNPad;
#pragma unroll
        for (int n = 0; n < kNPad; ++n) hin[n] = n < p.dstate ? __ldcg(hs + n) : 0.0f;
        correct_chain<IoT, BcT, kHasZ, kSoftplus, true>(p, chain, k, hin, lane);
    }
}

}  // namespace mamba
