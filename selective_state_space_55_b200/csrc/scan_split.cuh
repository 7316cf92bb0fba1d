// Selective-scan forward with two lanes per channel (sm_100a).
//
// The scan kernel of selective_scan.cuh gives each lane one channel, so a
// batch row of D channels makes D / 32 warps.  When the channel groups are
// fewer than the warps the GPU holds at once (8 x 4096 channels: 1024 groups
// for 2368 warp slots), each warp runs alone on its sub-partition most of the
// time and stalls on the latency of each step's dependent arithmetic.  This
// kernel halves the channels per warp: lane l holds channel l & 15 and the
// state entries 8 (l >> 4) .. 8 (l >> 4) + 7 of it (its "half"), so the same
// work spreads over twice as many warps.
//
// Nothing transcendental is formed twice.  Within each pair of steps a lane
// takes the softplus of one step and swaps it with its partner lane (one
// shuffle); each lane advances its 8 entries and forms its half of the
// readout C_t . h_t for every step; then the halves are exchanged (one
// shuffle per pair of steps) so that each lane finishes half of the steps:
// the sum of the halves, D u, the gate silu(z) and the store.  The MUFU work
// per element is that of the one-lane kernel.
//
// Scope: chained segments (mode 0) with outputs, the Euler input term and the
// (batch, dim, seqlen) layout; staging, handoff and bounded waits as in
// selective_scan.cuh, with tiles of 16 channel rows.
#pragma once

#include "selective_scan.cuh"

namespace mamba {

// Per-warp shared memory: two stages of u, delta, z (16 rows of 32 bytes
// each) and the raw B and C rows, at the same offsets as the one-lane
// layout's so that its B/C conversion serves both, then the fp32 B/C table
// and the mbarriers.
struct SplitLayout {
    static constexpr int kRows = 16;                              // channels per group
    static constexpr int kIoTile = kRows * kRowBytes;             // 512 bytes
    static constexpr int kOffU = 0;
    static constexpr int kOffDelta = kIoTile;
    static constexpr int kOffZ = 2 * kIoTile;
    static constexpr int kOffB = ScanLayout<1>::kOffB;
    static constexpr int kOffC = ScanLayout<1>::kOffC;
    static constexpr int kStage = kOffC + kBcRawBytes;
    static constexpr int kOffBcf = kScanStages * kStage;
    static constexpr int kOffBar = kOffBcf + kBcfBytes;
    static constexpr int kWarpSmem = ((kOffBar + 64 + 255) / 256) * 256;
    static constexpr int kWarps = 4;                                 // warps per CTA
    static constexpr int kCtaSmem = kWarps * kWarpSmem + 1024;       // + base alignment slack
    // Three CTAs per SM, so up to 168 registers: on 8 x 4096 channels (2048
    // warps) measured 1.2% faster than four CTAs at 128 registers, although
    // fewer warps are resident at once.
    static constexpr int kMinBlocks = 3;                             // CTAs per SM
    static constexpr int kWarpsPerSm = kWarps * kMinBlocks;
    static_assert(3 * kIoTile <= kOffB, "activation tiles overlap the B rows");
    static_assert(kStage % 256 == 0 && kWarpSmem % 256 == 0, "32-byte swizzle needs 256-byte tiles");
};

// One lane's half of one channel: entries 8 hf .. 8 hf + 7 as four pairs.
struct SplitChains {
    float2 h[4];
    float2 a2[4];      // A_d,n log2(e)
    float bias;
    float Dd;
};

// Element 2k + hf of a 16-byte vector (the step of a pair this lane takes).
template <typename IoT>
__device__ __forceinline__ float pair_elem(const uint4& v, int k, int hf);
template <>
__device__ __forceinline__ float pair_elem<__nv_bfloat16>(const uint4& v, int k, int hf) {
    const uint32_t w = k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
    return __uint_as_float(hf ? (w & 0xffff0000u) : (w << 16));
}
template <>
__device__ __forceinline__ float pair_elem<float>(const uint4& v, int k, int hf) {
    const uint32_t w = k == 0 ? (hf ? v.y : v.x) : (hf ? v.w : v.z);
    return __uint_as_float(w);
}

// Element hf * (V / 2) + k of a 16-byte vector of V values (a step of the
// half of the vector whose output this lane finishes).
template <typename IoT>
__device__ __forceinline__ float half_elem(const uint4& v, int k, int hf);
template <>
__device__ __forceinline__ float half_elem<__nv_bfloat16>(const uint4& v, int k, int hf) {
    const uint32_t w = k < 2 ? (hf ? v.z : v.x) : (hf ? v.w : v.y);
    return __uint_as_float((k & 1) ? (w & 0xffff0000u) : (w << 16));
}
template <>
__device__ __forceinline__ float half_elem<float>(const uint4& v, int k, int hf) {
    return __uint_as_float(k == 0 ? (hf ? v.z : v.x) : (hf ? v.w : v.y));
}

// One step of one lane's 8 entries; returns its half of C_t . h_t.
template <bool kExact>
__device__ __forceinline__ float split_step(const float* bc_row, int hf, float dt, float du,
                                            SplitChains& lc) {
    const float4* b4 = reinterpret_cast<const float4*>(bc_row + 8 * hf);
    const float4* c4 = reinterpret_cast<const float4*>(bc_row + 16 + 8 * hf);
    const float2 dt2 = make_float2(dt, dt);
    const float2 du2 = make_float2(du, du);
    float2 ya = make_float2(0.0f, 0.0f), yb = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const float4 Bq = b4[q];
        const float2 bq[2] = {make_float2(Bq.x, Bq.y), make_float2(Bq.z, Bq.w)};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int pi = 2 * q + half;
            const float2 x2 = __fmul2_rn(dt2, lc.a2[pi]);
            const float2 abar = exp2_pair<kExact>(x2);
            const float2 in = __fmul2_rn(du2, bq[half]);
            lc.h[pi] = __ffma2_rn(abar, lc.h[pi], in);
        }
        const float4 Cq = c4[q];
        const float2 c01 = make_float2(Cq.x, Cq.y);
        const float2 c23 = make_float2(Cq.z, Cq.w);
        if (q == 0) {
            ya = __fmul2_rn(c01, lc.h[0]);
            yb = __fmul2_rn(c23, lc.h[1]);
        } else {
            ya = __ffma2_rn(c01, lc.h[2], ya);
            yb = __ffma2_rn(c23, lc.h[3], yb);
        }
    }
    const float2 t = __fadd2_rn(ya, yb);
    return t.x + t.y;
}

// The valid steps (nsteps <= T) of one staged tile, one 16-byte vector (V
// steps) at a time.  out_row is null for channels past dim (both lanes of a
// channel agree); every lane takes part in the shuffles.
template <typename IoT, bool kHasZ, bool kSoftplus>
__device__ __forceinline__ void compute_tile_split(const uint8_t* st, const float* bcf, int lane,
                                                   int nsteps, SplitChains& lc, IoT* out_row,
                                                   bool vec_out) {
    using Lay = SplitLayout;
    constexpr int V = 16 / (int)sizeof(IoT);          // steps per 16-byte vector
    constexpr int H = V / 2;                          // steps of a vector this lane finishes
    constexpr int T = kRowBytes / (int)sizeof(IoT);   // steps per tile
    constexpr bool kExact = sizeof(IoT) == 4;
    const int r = lane & 15;
    const int hf = lane >> 4;
#pragma unroll 1
    for (int cv = 0; cv < T / V; ++cv) {
        const int base = cv * V;
        if (base >= nsteps) break;
        const uint32_t so = swz32(r, 16u * cv);
        const uint4 ur = *reinterpret_cast<const uint4*>(st + Lay::kOffU + so);
        const uint4 dr = *reinterpret_cast<const uint4*>(st + Lay::kOffDelta + so);
        uint4 zr = make_uint4(0u, 0u, 0u, 0u);
        if (kHasZ) zr = *reinterpret_cast<const uint4*>(st + Lay::kOffZ + so);
        const int steps = min(V, nsteps - base);
        // Delta of every step: this lane forms step 2k + hf of each pair, its
        // partner the other one
        float dtv[V];
#pragma unroll
        for (int k = 0; k < H; ++k) {
            const float s = pair_elem<IoT>(dr, k, hf) + lc.bias;
            const float mine = kSoftplus ? (kExact ? softplus_f32(s) : softplus_lg2(s)) : s;
            const float other = __shfl_xor_sync(0xffffffffu, mine, 16);
            dtv[2 * k] = hf ? other : mine;
            dtv[2 * k + 1] = hf ? mine : other;
        }
        // this lane's 8 entries over the vector's steps, and its half of each readout
        float yh[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            yh[j] = 0.0f;
            if (steps == V || j < steps)
                yh[j] = split_step<kExact>(bcf + (base + j) * 32, hf, dtv[j],
                                           dtv[j] * vec_elem<IoT>(ur, j), lc);
        }
        // swap halves: this lane finishes steps hf H .. hf H + H - 1 of the vector
        float yo[H];
#pragma unroll
        for (int k = 0; k < H; ++k) {
            const float send = hf ? yh[k] : yh[H + k];
            const float mine = hf ? yh[H + k] : yh[k];
            yo[k] = mine + __shfl_xor_sync(0xffffffffu, send, 16);
        }
        if (out_row == nullptr) continue;
        const int j0 = hf * H;
        float o[H];
#pragma unroll
        for (int k = 0; k < H; ++k) {
            float v = fmaf(lc.Dd, half_elem<IoT>(ur, k, hf), yo[k]);
            if (kHasZ) {
                const float zk = half_elem<IoT>(zr, k, hf);
                v *= kExact ? silu_f32(zk) : silu_tanh(zk);
            }
            o[k] = v;
        }
        if (steps == V && vec_out) {   // H values = 8 bytes, 8-byte aligned
            uint2 w;
            if constexpr (sizeof(IoT) == 2) {
                w = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
            } else {
                w = make_uint2(__float_as_uint(o[0]), __float_as_uint(o[1]));
            }
            *reinterpret_cast<uint2*>(out_row + base + j0) = w;
        } else {
#pragma unroll
            for (int k = 0; k < H; ++k)
                if (j0 + k < steps) DType<IoT>::store(out_row + base + j0 + k, o[k]);
        }
    }
}

// Fill one stage with plain loads (any stride or alignment); rows beyond dim
// and steps beyond seqlen read as zero, as TMA's out-of-bounds fill does.
template <typename IoT, bool kNeedZ>
__device__ __forceinline__ void portable_stage_split(const ScanParams& p, uint8_t* st, float* bcf,
                                                     int lane, int64_t b, int64_t d0, int64_t t0) {
    using Lay = SplitLayout;
    constexpr int ES = (int)sizeof(IoT);
    constexpr int T = kRowBytes / ES;
    const IoT* u = static_cast<const IoT*>(p.u);
    const IoT* dl = static_cast<const IoT*>(p.delta);
    const IoT* zz = static_cast<const IoT*>(p.z);
    for (int idx = lane; idx < Lay::kRows * T; idx += 32) {
        const int r = idx / T;
        const int j = idx % T;
        const int64_t d = d0 + r;
        const int64_t t = t0 + j;
        const bool in = d < p.dim && t < p.seqlen;
        const int64_t off = (b * p.dim + d) * p.seqlen + t;
        const uint32_t so = swz32(r, j * ES);
        const IoT zero = IoT(0.0f);
        *reinterpret_cast<IoT*>(st + Lay::kOffU + so) = in ? u[off] : zero;
        *reinterpret_cast<IoT*>(st + Lay::kOffDelta + so) = in ? dl[off] : zero;
        if (kNeedZ) *reinterpret_cast<IoT*>(st + Lay::kOffZ + so) = in ? zz[off] : zero;
    }
    const int which = lane >> 4;
    const int n = lane & 15;
    const bool live = n < p.dstate;
    const void* src = which ? p.C : p.B;
    for (int k = 0; k < T; ++k) {
        const int j = (k + lane) & (T - 1);
        const int64_t t = t0 + j;
        float v = 0.0f;
        if (live && t < p.seqlen) {
            const int64_t off = (b * p.dstate + n) * p.seqlen + t;
            v = p.bc_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(src)[off])
                          : static_cast<const float*>(src)[off];
        }
        bcf[j * 32 + lane] = v;
    }
}

// Run time steps [t_begin, t_end) of one group from lc.h (chained mode, with
// outputs).  `seq` counts the tiles this warp has consumed (stage and
// mbarrier parity).  Returns false if a staged tile never arrived (the warp
// has then waited, bounded, for its copies in flight).
template <typename IoT, bool kHasZ, bool kSoftplus>
__device__ __forceinline__ bool run_segment_split(const ScanParams& p, const TmaMaps& maps,
                                                  uint8_t* wsm, int lane, int64_t b, int64_t d0,
                                                  int64_t t_begin, int64_t t_end, SplitChains& lc,
                                                  IoT* out_row, uint32_t& seq) {
    using Lay = SplitLayout;
    constexpr int T = kRowBytes / (int)sizeof(IoT);
    uint64_t* bars = reinterpret_cast<uint64_t*>(wsm + Lay::kOffBar);
    float* bcf = reinterpret_cast<float*>(wsm + Lay::kOffBcf);
    const int ntiles = (int)((t_end - t_begin + T - 1) / T);
    const uint32_t bc_bytes = (uint32_t)(p.dstate * T * (p.bc_bf16 ? 2 : 4));
    const uint32_t stage_tx = (uint32_t)((kHasZ ? 3 : 2) * Lay::kIoTile) + 2u * bc_bytes;

    auto issue = [&](int i) {
        const uint32_t s = (seq + (uint32_t)i) % kScanStages;
        uint8_t* st = wsm + s * Lay::kStage;
        const int t0 = (int)(t_begin + (int64_t)i * T);
        const uint32_t bar = smem_u32(&bars[s]);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, stage_tx);
        tma_load_3d(smem_u32(st + Lay::kOffU), maps.u, t0, (int)d0, (int)b, bar);
        tma_load_3d(smem_u32(st + Lay::kOffDelta), maps.delta, t0, (int)d0, (int)b, bar);
        if (kHasZ) tma_load_3d(smem_u32(st + Lay::kOffZ), maps.z, t0, (int)d0, (int)b, bar);
        tma_load_3d(smem_u32(st + Lay::kOffB), maps.B, t0, 0, (int)b, bar);
        tma_load_3d(smem_u32(st + Lay::kOffC), maps.C, t0, 0, (int)b, bar);
    };

    if (p.use_tma && lane == 0)
        for (int i = 0; i < kScanStages && i < ntiles; ++i) issue(i);
    __syncwarp();

    for (int i = 0; i < ntiles; ++i) {
        const uint32_t sq = seq + (uint32_t)i;
        uint8_t* st = wsm + (sq % kScanStages) * Lay::kStage;
        const int64_t t0 = t_begin + (int64_t)i * T;
        const int nsteps = (int)min((int64_t)T, t_end - t0);
        if (p.use_tma) {
            bool ok = mbar_wait_bounded(smem_u32(&bars[sq % kScanStages]), (sq / kScanStages) & 1u);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                if (lane == 0) {
                    record_device_error(MAMBA_ERR_TIMEOUT);
                    for (int j = i; j < ntiles && j < i + kScanStages; ++j) {
                        const uint32_t sj = seq + (uint32_t)j;
                        (void)mbar_wait_bounded(smem_u32(&bars[sj % kScanStages]),
                                                (sj / kScanStages) & 1u);
                    }
                }
                __syncwarp();
                return false;
            }
            convert_bc<1, T, true>(st, bcf, lane, p.dstate, p.bc_bf16 != 0);
        } else {
            portable_stage_split<IoT, kHasZ>(p, st, bcf, lane, b, d0, t0);
        }
        __syncwarp();
        compute_tile_split<IoT, kHasZ, kSoftplus>(st, bcf, lane, nsteps, lc,
                                                  out_row ? out_row + (t0 - t_begin) : nullptr,
                                                  p.vec_out != 0);
        __syncwarp();
        if (p.use_tma && lane == 0 && i + kScanStages < ntiles) issue(i + kScanStages);
    }
    seq += (uint32_t)ntiles;
    return true;
}

template <typename IoT, bool kHasZ, bool kSoftplus>
__global__ void __launch_bounds__(SplitLayout::kWarps * 32, SplitLayout::kMinBlocks)
    selective_scan_fwd_split_kernel(const __grid_constant__ ScanParams p,
                                    const __grid_constant__ CUtensorMap tm_u,
                                    const __grid_constant__ CUtensorMap tm_delta,
                                    const __grid_constant__ CUtensorMap tm_z,
                                    const __grid_constant__ CUtensorMap tm_B,
                                    const __grid_constant__ CUtensorMap tm_C) {
    using Lay = SplitLayout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int hf = lane >> 4;
    uint8_t* wsm = smem + warp * Lay::kWarpSmem;
    const TmaMaps maps{&tm_u, &tm_delta, &tm_z, &tm_B, &tm_C};

    if (p.use_tma && lane == 0) {
        uint64_t* bars = reinterpret_cast<uint64_t*>(wsm + Lay::kOffBar);
        for (int s = 0; s < kScanStages; ++s) mbar_init(smem_u32(&bars[s]), 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_u);
        prefetch_tensormap(&tm_delta);
        prefetch_tensormap(&tm_B);
    }
    __syncwarp();

    uint32_t seq = 0;
    for (;;) {
        unsigned int item = 0;
        if (lane == 0) item = atomicAdd(p.counter, 1u);
        item = __shfl_sync(0xffffffffu, item, 0);
        if ((int64_t)item >= p.items) break;
        const int64_t g = item % p.groups;
        const int64_t k = item / p.groups;
        const int64_t b = g / p.groups_per_batch;
        const int64_t d0 = (g % p.groups_per_batch) * Lay::kRows;
        const int64_t t_begin = k * p.seg_len;
        const int64_t t_end = min(t_begin + p.seg_len, p.seqlen);
        const int64_t d = d0 + (lane & 15);
        const bool valid = d < p.dim;
        const int64_t chain = b * p.dim + d;

        SplitChains lc;
#pragma unroll
        for (int pi = 0; pi < 4; ++pi) {
            const int n = 8 * hf + 2 * pi;
            const bool in0 = valid && n < p.dstate;
            const bool in1 = valid && n + 1 < p.dstate;
            const float a0 = in0 ? p.A[d * p.dstate + n] : 0.0f;
            const float a1 = in1 ? p.A[d * p.dstate + n + 1] : 0.0f;
            lc.a2[pi] = make_float2(a0 * kLog2e, a1 * kLog2e);
            const float* h0 = (k == 0 && p.h0 != nullptr) ? p.h0 + chain * p.dstate : nullptr;
            lc.h[pi] = make_float2((h0 != nullptr && in0) ? h0[n] : 0.0f,
                                   (h0 != nullptr && in1) ? h0[n + 1] : 0.0f);
        }
        lc.bias = (valid && p.delta_bias != nullptr) ? p.delta_bias[d] : 0.0f;
        lc.Dd = (valid && p.D != nullptr) ? p.D[d] : 0.0f;

        if (k > 0) {   // wait for segment k-1 of this group, then take over its state
            bool ok = true;
            if (lane == 0) {
                ok = false;
                for (uint32_t i = 0; i < p.flag_poll_limit; ++i) {
                    if (ld_acquire_gpu(p.flags + g) >= (unsigned int)k) {
                        ok = true;
                        break;
                    }
                    __nanosleep(1000);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                if (lane == 0) record_device_error(MAMBA_ERR_TIMEOUT);
                break;
            }
            (void)ld_acquire_gpu(p.flags + g);
            if (valid) {
                const float4* src = reinterpret_cast<const float4*>(p.carry + chain * kNPad + 8 * hf);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const float4 v = __ldcg(src + q);
                    lc.h[2 * q] = make_float2(v.x, v.y);
                    lc.h[2 * q + 1] = make_float2(v.z, v.w);
                }
            }
        }

        IoT* out_row = (valid && p.out != nullptr)
                           ? static_cast<IoT*>(p.out) + chain * p.seqlen + t_begin : nullptr;
        if (!run_segment_split<IoT, kHasZ, kSoftplus>(p, maps, wsm, lane, b, d0, t_begin, t_end,
                                                      lc, out_row, seq))
            break;

        if (k < p.nseg - 1) {   // hand the state on
            if (valid) {
                float4* dst = reinterpret_cast<float4*>(p.carry + chain * kNPad + 8 * hf);
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    __stcg(dst + q, make_float4(lc.h[2 * q].x, lc.h[2 * q].y, lc.h[2 * q + 1].x,
                                                lc.h[2 * q + 1].y));
            }
            __threadfence();
            __syncwarp();
            if (lane == 0 && !p.withhold_handoff) st_release_gpu(p.flags + g, (unsigned int)(k + 1));
        } else if (valid && p.last_state != nullptr) {
            float* ls = p.last_state + chain * p.dstate;
#pragma unroll
            for (int pi = 0; pi < 4; ++pi) {
                const int n = 8 * hf + 2 * pi;
                if (n < p.dstate) ls[n] = lc.h[pi].x;
                if (n + 1 < p.dstate) ls[n + 1] = lc.h[pi].y;
            }
        }
    }
}

}  // namespace mamba
