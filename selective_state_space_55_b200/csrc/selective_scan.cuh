// Selective-scan forward kernel (sm_100a).
//
// Work decomposition.  One warp owns 32 consecutive channels of one batch row
// (a "group") for one contiguous range of time steps (a "segment").  Lane l
// owns channel d = d0 + l: its 16 state values h_n and the 16 factors
// A_d,n * log2(e) live in registers for the whole segment, so the state never
// touches HBM ("Mamba 与状态空间模型", section 在芯片上扫过去: discretise and recur
// on chip, write only the output).  Each time step costs 16 MUFU ex2 for
// Abar = 2^(Delta * A log2 e), four fp32 operations per state entry, and the
// softplus / silu of the step.
//
// Scheduling.  The grid is persistent (as many CTAs as stay resident) and
// every warp pulls (segment k, group g) work items from a global counter in
// segment-major order, so the load balances across all SMs whatever the
// number of groups.  Two ways to split a sequence into K segments:
//
//  * chained (mode 0): item (k, g) starts from the state item (k-1, g) left in
//    an L2-resident carry buffer.  Item k-1 of the same group was dequeued G
//    items earlier, so with G >= resident warps it has normally finished and
//    the wait is free.  The handoff is a release/acquire flag per group; the
//    wait is bounded and reports MAMBA_ERR_TIMEOUT through the device status
//    word instead of hanging.  No work is repeated.
//  * parallel (modes 1, 2; few channels, very long sequences): pass A runs
//    segments 0..K-2 independently: segment 0 writes its outputs and end state,
//    segments k >= 1 only their end state from a zero start and the sum of
//    Delta.  Pass B runs segments 1..K-1: each folds the earlier segments'
//    (exp(A sum Delta), end state) pairs into its true start state, then
//    recomputes its outputs.  The fold applies the associative combine
//    (P1, h1) then (P2, h2) -> (P1 P2, P2 h1 + h2) of the parallel scan
//    ("Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
//    section 硬件效率; "Mamba 与状态空间模型", section 在芯片上扫过去).
//
// Staging.  Per warp, a two-stage ring in shared memory holds tiles of
// T = 32 bytes / sizeof(io) time steps of the warp's 32 channel rows of u,
// delta and z (TMA 3-D tiles with 32-byte swizzle, so each lane's 16-byte reads
// of its own row are conflict free; L2 promotion fetches whole 128-byte lines
// so the next tiles of a row hit L2) and the B and C rows of the batch (TMA).
// Once a tile lands the warp converts B and C to an fp32 table
// bcf[t][B0..15 C0..15] that every lane reads with broadcast 16-byte loads.
// Without TMA (odd strides or MAMBA_FLAG_NO_TMA) plain loads fill the same
// tiles.  About 12 KB of shared memory and at most 128 registers per warp let
// 16 warps share an SM.
#pragma once

#include "ssm_device.cuh"

namespace mamba {

constexpr int kScanWarps = 4;              // warps per CTA (each an independent worker)
#ifndef MAMBA_SCAN_MIN_BLOCKS
#define MAMBA_SCAN_MIN_BLOCKS 4
#endif
constexpr int kScanMinBlocks = MAMBA_SCAN_MIN_BLOCKS;   // CTAs per SM the kernel is compiled for
constexpr int kScanStages = 2;             // tiles in flight per warp
constexpr int kRowBytes = 32;              // bytes of one channel row in a tile
constexpr int kGroupRows = 32;             // channels per warp
constexpr int kNPad = 16;                  // compiled state size (smaller N is zero-padded)
constexpr int kMaxTile = kRowBytes / 2;    // time steps per tile for 2-byte inputs
constexpr int kIoTileBytes = kGroupRows * kRowBytes;        // 1024
constexpr int kBcRawBytes = kNPad * kMaxTile * 4;           // 16 rows of up to 64 bytes
constexpr int kOffU = 0;
constexpr int kOffDelta = kIoTileBytes;
constexpr int kOffZ = 2 * kIoTileBytes;
constexpr int kOffB = 3 * kIoTileBytes;
constexpr int kOffC = 3 * kIoTileBytes + kBcRawBytes;
constexpr int kStageBytes = 3 * kIoTileBytes + 2 * kBcRawBytes;   // 5120
constexpr int kBcfBytes = kMaxTile * 32 * 4;                      // [T][32] fp32
constexpr int kBarOffset = kScanStages * kStageBytes + kBcfBytes;
constexpr int kWarpSmemBytes = ((kBarOffset + 64 + 255) / 256) * 256;
constexpr int kScanSmemBytes = kScanWarps * kWarpSmemBytes + 1024;  // + base alignment slack
constexpr int kScanWarpsPerSm = kScanWarps * kScanMinBlocks;

// Workspace layout (bytes from the start).
constexpr size_t kWsCounters = 0;          // uint32 [2] dequeue counters
constexpr size_t kWsFlags = 256;           // uint32 [groups] finished segments per group

enum ScanMode { kModeChained = 0, kModePassA = 1, kModePassB = 2 };

struct ScanParams {
    const void* u;
    const void* delta;
    const void* z;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* delta_bias;
    void* out;
    float* last_state;
    unsigned int* counter;   // dequeue counter of this launch
    unsigned int* flags;     // [groups] (chained mode)
    float* carry;            // [chains][16] (chained mode)
    float* ws_h;             // [K-1][chains][16] (parallel mode)
    float* ws_sdt;           // [K-1][chains]     (parallel mode)
    int64_t batch, dim, seqlen;
    int64_t groups_per_batch, groups, chains;
    int64_t seg_len;
    int64_t items;
    int dstate;
    int nseg;
    int mode;
    int use_tma;
    int bc_bf16;
    int vec_out;             // 16-byte output stores are aligned
    unsigned int flag_poll_limit;   // chained mode: polls (~1 us each) before a wait gives up
    int withhold_handoff;    // test only: segments never publish their state (waits time out)
};

// Byte offset of (row r, byte x of the row) in a 32-byte-row tile written by
// TMA with 32-byte swizzle: address bit 4 is XORed with bit 7.
__device__ __forceinline__ uint32_t swz32(uint32_t r, uint32_t x) {
    const uint32_t o = r * kRowBytes + x;
    return o ^ (((o >> 7) & 1u) << 4);
}

__device__ __forceinline__ void kahan_add(float& sum, float& comp, float v) {
    const float y = v - comp;
    const float t = sum + y;
    comp = (t - sum) - y;
    sum = t;
}

// One time step for one lane: advance the 16 states, return y (kOut).
// kExact selects exp2_near_one_exact for Abar (fp32 input/output path).
template <bool kOut, bool kExact>
__device__ __forceinline__ float scan_step(const float* bc_row, float dt, float du,
                                           float (&h)[kNPad], const float (&a2)[kNPad]) {
    const float4* bc = reinterpret_cast<const float4*>(bc_row);
    float yq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 Bq = bc[q];
        const float b4[4] = {Bq.x, Bq.y, Bq.z, Bq.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int n = 4 * q + i;
            const float x = dt * a2[n];
            const float abar = kExact ? exp2_near_one_exact(x) : ex2_approx(x);
            h[n] = fmaf(abar, h[n], du * b4[i]);
        }
        if (kOut) {
            const float4 Cq = bc[4 + q];
            float y = Cq.x * h[4 * q];
            y = fmaf(Cq.y, h[4 * q + 1], y);
            y = fmaf(Cq.z, h[4 * q + 2], y);
            y = fmaf(Cq.w, h[4 * q + 3], y);
            yq[q] = y;
        }
    }
    return kOut ? (yq[0] + yq[1]) + (yq[2] + yq[3]) : 0.0f;
}

// Element j of a 16-byte vector holding 8 bf16 or 4 fp32 values, as fp32.
template <typename IoT>
__device__ __forceinline__ float vec_elem(const uint4& v, int j);
template <>
__device__ __forceinline__ float vec_elem<__nv_bfloat16>(const uint4& v, int j) {
    const uint32_t w = j < 2 ? v.x : j < 4 ? v.y : j < 6 ? v.z : v.w;
    return (j & 1) ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
}
template <>
__device__ __forceinline__ float vec_elem<float>(const uint4& v, int j) {
    return __uint_as_float(j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w);
}

// Packs the outputs of one 16-byte chunk as they are produced.
template <typename IoT> struct OutPack;
template <> struct OutPack<__nv_bfloat16> {
    uint32_t w[4];
    float prev;
    __device__ __forceinline__ void put(int j, float y) {
        if (j & 1) w[j >> 1] = pack_bf16x2(prev, y);
        else prev = y;
    }
    __device__ __forceinline__ uint4 vec() const { return make_uint4(w[0], w[1], w[2], w[3]); }
};
template <> struct OutPack<float> {
    uint32_t w[4];
    __device__ __forceinline__ void put(int j, float y) { w[j] = __float_as_uint(y); }
    __device__ __forceinline__ uint4 vec() const { return make_uint4(w[0], w[1], w[2], w[3]); }
};

// Process the `nsteps` (<= T) valid time steps of one staged tile.  The
// 16-byte vectors of u, delta and z stay packed and are unpacked step by
// step, which keeps the kernel within 128 registers.
template <typename IoT, bool kHasZ, bool kSoftplus, bool kOut>
__device__ __forceinline__ void compute_tile(const uint8_t* st, const float* bcf, int lane,
                                             int nsteps, float (&h)[kNPad],
                                             const float (&a2)[kNPad], float bias, float Dd,
                                             IoT* out_row, bool vec_out, float& sdt,
                                             float& sdt_c) {
    constexpr int V = 16 / (int)sizeof(IoT);          // steps per 16-byte vector
    constexpr int T = kRowBytes / (int)sizeof(IoT);   // steps per tile
    constexpr bool kExact = sizeof(IoT) == 4;
#pragma unroll 1
    for (int c = 0; c < T / V; ++c) {
        const int base = c * V;
        if (base >= nsteps) break;
        const uint32_t so = swz32(lane, 16u * c);
        const uint4 ur = *reinterpret_cast<const uint4*>(st + kOffU + so);
        const uint4 dr = *reinterpret_cast<const uint4*>(st + kOffDelta + so);
        uint4 zr = make_uint4(0u, 0u, 0u, 0u);
        if (kHasZ && kOut) zr = *reinterpret_cast<const uint4*>(st + kOffZ + so);
        const int steps = min(V, nsteps - base);
        const bool whole = steps == V && vec_out && out_row != nullptr;
        OutPack<IoT> pk;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            if (steps == V || j < steps) {
                const float uj = vec_elem<IoT>(ur, j);
                const float s = vec_elem<IoT>(dr, j) + bias;
                const float dt = kSoftplus ? softplus_f32(s) : s;
                const float y = scan_step<kOut, kExact>(bcf + (base + j) * 32, dt, dt * uj, h, a2);
                if (kOut) {
                    float yo = fmaf(Dd, uj, y);
                    if (kHasZ) yo *= silu_f32(vec_elem<IoT>(zr, j));
                    if (whole)
                        pk.put(j, yo);
                    else if (out_row != nullptr)
                        DType<IoT>::store(out_row + base + j, yo);
                } else {
                    kahan_add(sdt, sdt_c, dt);
                }
            }
        }
        if (kOut && whole) *reinterpret_cast<uint4*>(out_row + base) = pk.vec();
    }
}

// Convert the raw B (and C) rows of a TMA-staged tile into the fp32 table
// bcf[t][32] = (B_0..B_15, C_0..C_15) of each step.  Lane l handles row
// l & 15 of B (l < 16) or C; rows n >= dstate read as zero.
template <int T, bool kNeedC>
__device__ __forceinline__ void convert_bc(const uint8_t* st, float* bcf, int lane, int dstate,
                                           bool bc_bf16) {
    const int which = lane >> 4;
    const int n = lane & 15;
    const bool live = n < dstate && (which == 0 || kNeedC);
    const uint8_t* raw = st + (which ? kOffC : kOffB);
#pragma unroll
    for (int k = 0; k < T; ++k) {
        const int j = (k + lane) & (T - 1);
        float v = 0.0f;
        if (live) {
            if (bc_bf16)
                v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(raw)[n * T + j]);
            else
                v = reinterpret_cast<const float*>(raw)[n * T + j];
        }
        bcf[j * 32 + lane] = v;
    }
}

// Fill one stage with plain loads (any stride or alignment).  Rows beyond
// dim and steps beyond seqlen read as zero, as TMA's out-of-bounds fill does.
template <typename IoT, bool kNeedZ, bool kNeedC>
__device__ __forceinline__ void portable_stage(const ScanParams& p, uint8_t* st, float* bcf,
                                               int lane, int64_t b, int64_t d0, int64_t t0) {
    constexpr int ES = (int)sizeof(IoT);
    constexpr int T = kRowBytes / ES;
    const IoT* u = static_cast<const IoT*>(p.u);
    const IoT* dl = static_cast<const IoT*>(p.delta);
    const IoT* zz = static_cast<const IoT*>(p.z);
    for (int idx = lane; idx < kGroupRows * T; idx += 32) {
        const int r = idx / T;
        const int j = idx % T;
        const int64_t d = d0 + r;
        const int64_t t = t0 + j;
        const bool in = d < p.dim && t < p.seqlen;
        const int64_t off = (b * p.dim + d) * p.seqlen + t;
        const uint32_t so = swz32(r, j * ES);
        const IoT zero = IoT(0.0f);
        *reinterpret_cast<IoT*>(st + kOffU + so) = in ? u[off] : zero;
        *reinterpret_cast<IoT*>(st + kOffDelta + so) = in ? dl[off] : zero;
        if (kNeedZ) *reinterpret_cast<IoT*>(st + kOffZ + so) = in ? zz[off] : zero;
    }
    const int which = lane >> 4;
    const int n = lane & 15;
    const bool live = n < p.dstate && (which == 0 || kNeedC);
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

struct TmaMaps {
    const CUtensorMap* u;
    const CUtensorMap* delta;
    const CUtensorMap* z;
    const CUtensorMap* B;
    const CUtensorMap* C;
};

// Run time steps [t_begin, t_end) of one group, starting from h.  `seq`
// counts the tiles this warp has consumed (it fixes each tile's stage and
// mbarrier parity across items).  Returns false if a staged tile never
// arrived (the warp has then waited, bounded, for its copies in flight).
template <typename IoT, bool kHasZ, bool kSoftplus, bool kOut>
__device__ __forceinline__ bool run_segment(const ScanParams& p, const TmaMaps& maps, uint8_t* wsm,
                                            int lane, int64_t b, int64_t d0, int64_t t_begin,
                                            int64_t t_end, float (&h)[kNPad],
                                            const float (&a2)[kNPad], float bias, float Dd,
                                            IoT* out_row, uint32_t& seq, float& sdt) {
    constexpr int T = kRowBytes / (int)sizeof(IoT);
    constexpr bool kNeedZ = kHasZ && kOut;
    uint64_t* bars = reinterpret_cast<uint64_t*>(wsm + kBarOffset);
    float* bcf = reinterpret_cast<float*>(wsm + kScanStages * kStageBytes);
    float sdt_c = 0.0f;

    const int ntiles = (int)((t_end - t_begin + T - 1) / T);
    const uint32_t bc_bytes = (uint32_t)(p.dstate * T * (p.bc_bf16 ? 2 : 4));
    const uint32_t stage_tx =
        (uint32_t)((kNeedZ ? 3 : 2) * kIoTileBytes) + (kOut ? 2u : 1u) * bc_bytes;

    auto issue = [&](int i) {
        const uint32_t s = (seq + (uint32_t)i) % kScanStages;
        uint8_t* st = wsm + s * kStageBytes;
        const int t0 = (int)(t_begin + (int64_t)i * T);
        const uint32_t bar = smem_u32(&bars[s]);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, stage_tx);
        tma_load_3d(smem_u32(st + kOffU), maps.u, t0, (int)d0, (int)b, bar);
        tma_load_3d(smem_u32(st + kOffDelta), maps.delta, t0, (int)d0, (int)b, bar);
        if (kNeedZ) tma_load_3d(smem_u32(st + kOffZ), maps.z, t0, (int)d0, (int)b, bar);
        tma_load_3d(smem_u32(st + kOffB), maps.B, t0, 0, (int)b, bar);
        if (kOut) tma_load_3d(smem_u32(st + kOffC), maps.C, t0, 0, (int)b, bar);
    };

    if (p.use_tma && lane == 0)
        for (int i = 0; i < kScanStages && i < ntiles; ++i) issue(i);
    __syncwarp();

    for (int i = 0; i < ntiles; ++i) {
        const uint32_t sq = seq + (uint32_t)i;
        uint8_t* st = wsm + (sq % kScanStages) * kStageBytes;
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
            convert_bc<T, kOut>(st, bcf, lane, p.dstate, p.bc_bf16 != 0);
        } else {
            portable_stage<IoT, kNeedZ, kOut>(p, st, bcf, lane, b, d0, t0);
        }
        __syncwarp();
        compute_tile<IoT, kHasZ, kSoftplus, kOut>(st, bcf, lane, nsteps, h, a2, bias, Dd,
                                                  out_row ? out_row + (t0 - t_begin) : nullptr,
                                                  p.vec_out != 0, sdt, sdt_c);
        __syncwarp();
        if (p.use_tma && lane == 0 && i + kScanStages < ntiles) issue(i + kScanStages);
    }
    seq += (uint32_t)ntiles;
    return true;
}

__device__ __forceinline__ void store16(float* dst, const float (&h)[kNPad]) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        __stcg(d4 + q, make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]));
}

__device__ __forceinline__ void load16(const float* src, float (&h)[kNPad]) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 v = __ldcg(s4 + q);
        h[4 * q] = v.x; h[4 * q + 1] = v.y; h[4 * q + 2] = v.z; h[4 * q + 3] = v.w;
    }
}

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(unsigned int* p, unsigned int v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <typename IoT, bool kHasZ, bool kSoftplus>
__global__ void __launch_bounds__(kScanWarps * 32, kScanMinBlocks)
    selective_scan_fwd_kernel(const __grid_constant__ ScanParams p,
                              const __grid_constant__ CUtensorMap tm_u,
                              const __grid_constant__ CUtensorMap tm_delta,
                              const __grid_constant__ CUtensorMap tm_z,
                              const __grid_constant__ CUtensorMap tm_B,
                              const __grid_constant__ CUtensorMap tm_C) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    uint8_t* wsm = smem + warp * kWarpSmemBytes;
    const TmaMaps maps{&tm_u, &tm_delta, &tm_z, &tm_B, &tm_C};

    if (p.use_tma && lane == 0) {
        uint64_t* bars = reinterpret_cast<uint64_t*>(wsm + kBarOffset);
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
        const int64_t k = (p.mode == kModePassB ? 1 : 0) + item / p.groups;
        const int64_t b = g / p.groups_per_batch;
        const int64_t d0 = (g % p.groups_per_batch) * kGroupRows;
        const int64_t d = d0 + lane;
        const bool valid = d < p.dim;
        const int64_t chain = b * p.dim + d;
        const int64_t t_begin = k * p.seg_len;
        const int64_t t_end = min(t_begin + p.seg_len, p.seqlen);

        float a2[kNPad];
#pragma unroll
        for (int n = 0; n < kNPad; ++n)
            a2[n] = (valid && n < p.dstate) ? p.A[d * p.dstate + n] * kLog2e : 0.0f;
        const float bias = (valid && p.delta_bias != nullptr) ? p.delta_bias[d] : 0.0f;
        const float Dd = (valid && p.D != nullptr) ? p.D[d] : 0.0f;

        float h[kNPad];
#pragma unroll
        for (int n = 0; n < kNPad; ++n) h[n] = 0.0f;

        if (p.mode == kModeChained && k > 0) {
            // Wait for segment k-1 of this group, then take over its state.
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
            if (valid) load16(p.carry + chain * kNPad, h);
        } else if (p.mode == kModePassB && valid) {
            // True start state of segment k: fold the end states of 0..k-1.
            load16(p.ws_h + chain * kNPad, h);
            for (int64_t j = 1; j < k; ++j) {
                const float sj = __ldcg(p.ws_sdt + j * p.chains + chain);
                float hj[kNPad];
                load16(p.ws_h + (j * p.chains + chain) * kNPad, hj);
#pragma unroll
                for (int n = 0; n < kNPad; ++n) {
                    const float x = a2[n] * sj;
                    const float decay = sizeof(IoT) == 4 ? exp2_near_one_exact(x) : ex2_approx(x);
                    h[n] = fmaf(decay, h[n], hj[n]);
                }
            }
        }

        IoT* out_row = valid ? static_cast<IoT*>(p.out) + chain * p.seqlen + t_begin : nullptr;
        float sdt = 0.0f;
        bool ok;
        if (p.mode == kModePassA && k > 0)
            ok = run_segment<IoT, kHasZ, kSoftplus, false>(p, maps, wsm, lane, b, d0, t_begin, t_end,
                                                           h, a2, bias, Dd, nullptr, seq, sdt);
        else
            ok = run_segment<IoT, kHasZ, kSoftplus, true>(p, maps, wsm, lane, b, d0, t_begin, t_end,
                                                          h, a2, bias, Dd, out_row, seq, sdt);
        if (!ok) break;

        const bool last_seg = k == p.nseg - 1;
        if (p.mode == kModeChained) {
            if (!last_seg) {
                if (valid) store16(p.carry + chain * kNPad, h);
                __threadfence();
                __syncwarp();
                if (lane == 0 && !p.withhold_handoff)
                    st_release_gpu(p.flags + g, (unsigned int)(k + 1));
            }
        } else if (p.mode == kModePassA && valid) {
            store16(p.ws_h + (k * p.chains + chain) * kNPad, h);
            if (k >= 1) __stcg(p.ws_sdt + k * p.chains + chain, sdt);
        }
        if (last_seg && p.mode != kModePassA && valid && p.last_state != nullptr) {
            float* ls = p.last_state + chain * p.dstate;
#pragma unroll
            for (int n = 0; n < kNPad; ++n)
                if (n < p.dstate) ls[n] = h[n];
        }
    }
}

}  // namespace mamba
