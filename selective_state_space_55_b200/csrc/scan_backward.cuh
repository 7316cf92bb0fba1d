// Backward pass of the selective scan (sm_100a).
//
// Training back-propagates through the scan without keeping its per-step
// states: they are computed again from checkpoints ("Mamba 与状态空间模型",
// section 在芯片上扫过去).  With lambda_t = dLoss/dh_t, the adjoint runs in
// reverse time:
//
//   lambda_t   = C_t dy_t + Abar_t+1 lambda_t+1        (lambda_L-1 from dlast_state)
//   dC_t,n     = dy_t h_t,n          dB_t,n = lambda_t,n Delta_t u_t
//   dDelta_t   = sum_n lambda_t,n (B_t,n u_t + A_n Abar_t,n h_t-1,n)
//   dA_n      += lambda_t,n Delta_t Abar_t,n h_t-1,n
//   du_t       = D dy_t + Delta_t sum_n lambda_t,n B_t,n
//   dh_-1      = Abar_0 lambda_0
//
// with dy = dout silu(z), dz = dout y silu'(z) and the softplus derivative
// sigmoid(delta + bias) applied to dDelta.  With the zero-order-hold input
// term ("超越注意力：探索Mamba与状态空间模型", section 状态空间模型基础) the step is
// h_t = Abar_t h_t-1 + g_t B_t u_t with the gain g = expm1(Delta A) / A =
// Delta phi(Delta A) instead of Delta; then
//
//   dB_t,n     = lambda_t,n g_t,n u_t,   du_t = D dy_t + Delta_t sum_n lambda phi B
//   dDelta_t   = sum_n lambda_t,n (Abar_t,n B_t,n u_t + A_n Abar_t,n h_t-1,n)
//   dA_n      += lambda_t,n (Delta_t Abar_t,n h_t-1,n + dg/dA B_t,n u_t)
//
// with dg/dA = Delta (Abar - phi) / A, or its series Delta^2 (1/2 + x/3 + x^2/8
// + ...) (x = Delta A) where the difference would cancel.
//
// Layout of the work.  A first launch (the forward kernel in its checkpoint
// mode) stores the state before every block of kCkptSteps = 8 steps.  Then one
// warp owns 32 channels of one batch row for one segment, as in the forward,
// and walks the segment's 8-step blocks from the last to the first.  Segments
// run in reverse order: a segment starts from the lambda the later segment
// left in an L2-resident carry buffer (release/acquire flag, bounded wait).
// Within a block, for each quarter of the state (4 of the 16 entries) the lane
// recomputes the block's 8 states and their Abar from the checkpoint into
// registers, then runs the adjoint backwards over them, taking Abar_t h_t-1
// as h_t - Delta_t B_t u_t.  The lane's per-entry values (A log2 e, lambda,
// the running dA sum) wait in shared memory while other quarters run, so the
// quarter loop indexes registers statically and is emitted once.  A block
// shorter than 8 steps (the sequence's last) runs as a whole block whose
// missing steps have Delta = 0, u = dout = 0 and B = C = 0: they leave the
// state and lambda unchanged and contribute nothing.
//
// dB and dC sum over the channels of a batch row.  Per quarter and block each
// lane writes its 64 partials (8 steps x 4 entries x dB, dC) as one row of a
// per-warp table in shared memory; then each lane adds one pair of columns
// over the 32 rows and adds the two sums to global memory atomically.  dA, dD
// and the bias gradient are summed per lane over the segment and added once.
#pragma once

#include "selective_scan.cuh"

namespace mamba {

constexpr int kBwdWarps = 4;
constexpr int kBwdSteps = kCkptSteps;      // steps per block (one checkpoint each)

struct BwdParams {
    const void* u;
    const void* delta;
    const void* z;
    const void* dout;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* delta_bias;
    const float* dlast;        // (batch, dim, dstate) or null
    const float* ckpt;         // [chains][ckpt_tiles][16]
    void* du;
    void* ddelta;
    void* dz;
    float* dA;                 // (dim, dstate), accumulated
    float* dB;                 // (batch, dstate, seqlen), accumulated
    float* dC;
    float* dD;                 // (dim) or null, accumulated
    float* dbias;              // (dim) or null, accumulated
    float* dh0;                // (batch, dim, dstate) or null
    unsigned int* counter;
    unsigned int* flags;       // [groups] segments finished, counted from the end
    float* carry;              // [chains][16] lambda handed to the earlier segment
    int64_t batch, dim, seqlen, groups_per_batch, groups, chains, seg_len, items, ckpt_tiles;
    int dstate;
    int nseg;
    int softplus;
    int bc_bf16;
    int vec_ok;                // u, delta, z, dout, du, ddelta, dz all 16-byte aligned
    int bld;                   // those are (batch, seqlen, dim) (the kBld instances)
    int bc_vec;                // B and C rows 16-byte aligned
    unsigned int flag_poll_limit;
};

// kBwdSteps consecutive elements t0.. of a row as fp32 (zero past `n`); one
// 16-byte load when the row is 16-byte aligned at t0 and the block is whole.
template <typename T>
__device__ __forceinline__ void load_block(const T* row, int64_t t0, int n, bool vec,
                                           float (&v)[kBwdSteps]) {
    if (vec && n == kBwdSteps) {
        if constexpr (sizeof(T) == 2) {
            unpack16(*reinterpret_cast<const uint4*>(row + t0), v);
        } else {
            float a[4], b[4];
            unpack16(*reinterpret_cast<const uint4*>(row + t0), a);
            unpack16(*reinterpret_cast<const uint4*>(row + t0 + 4), b);
#pragma unroll
            for (int i = 0; i < 4; ++i) { v[i] = a[i]; v[4 + i] = b[i]; }
        }
        return;
    }
#pragma unroll
    for (int i = 0; i < kBwdSteps; ++i) v[i] = i < n ? DType<T>::load(row + t0 + i) : 0.0f;
}

template <typename T>
__device__ __forceinline__ void store_block(T* row, int64_t t0, int n, bool vec,
                                            const float (&v)[kBwdSteps]) {
    if (vec && n == kBwdSteps) {
        if constexpr (sizeof(T) == 2) {
            *reinterpret_cast<uint4*>(row + t0) = pack16(v);
        } else {
            const float a[4] = {v[0], v[1], v[2], v[3]}, b[4] = {v[4], v[5], v[6], v[7]};
            *reinterpret_cast<uint4*>(row + t0) = pack16(a);
            *reinterpret_cast<uint4*>(row + t0 + 4) = pack16(b);
        }
        return;
    }
#pragma unroll
    for (int i = 0; i < kBwdSteps; ++i)
        if (i < n) DType<T>::store(row + t0 + i, v[i]);
}

// kBwdSteps elements of one channel of a (batch, seqlen, dim) tensor, `step`
// elements apart (zero past `n`), and the matching stores.
template <typename T>
__device__ __forceinline__ void load_block_strided(const T* row, int64_t t0, int n, int64_t step,
                                                   float (&v)[kBwdSteps]) {
#pragma unroll
    for (int i = 0; i < kBwdSteps; ++i) v[i] = i < n ? DType<T>::load(row + (t0 + i) * step) : 0.0f;
}

template <typename T>
__device__ __forceinline__ void store_block_strided(T* row, int64_t t0, int n, int64_t step,
                                                    const float (&v)[kBwdSteps]) {
#pragma unroll
    for (int i = 0; i < kBwdSteps; ++i)
        if (i < n) DType<T>::store(row + (t0 + i) * step, v[i]);
}

// 16-byte asynchronous copy global -> shared (L2 only), and its groups.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)),
                 "l"(reinterpret_cast<uint64_t>(gmem_src))
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One lane's inputs of one 8-step block, staged by cp.async: its rows of u,
// delta, z and dout, its row of B (lanes 0..15) or C (16..31), and the
// checkpointed state.  Each lane reads back only what it copied.
template <typename IoT, typename BcT>
struct BwdStage {
    static constexpr int kIoRow = kBwdSteps * (int)sizeof(IoT);    // 16 or 32 bytes
    static constexpr int kBcRow = kBwdSteps * (int)sizeof(BcT);
    uint4 io[4][32][kIoRow / 16];
    uint4 bc[32][kBcRow / 16];
    uint4 ck[32][4];
};

// Per warp: two stages, the B/C table of one block, the lanes' per-entry
// values in quarters (A log2(e), lambda, the dA sum and, for the zero-order
// hold, 1 / A), and the dB/dC partials of one quarter of one block.  Each lane
// reads and writes only its own column of the per-entry values.
constexpr int kEntA2 = 0, kEntLam = 1, kEntDA = 2, kEntInvA = 3, kEntRows = 4;
// One lane's row of partials: 8 steps x (4 dB + 4 dC), padded to 68 floats so
// that the lanes' 16-byte stores of one step fall in distinct banks.
constexpr int kRedStride = 2 * 4 * kBwdSteps + 4;

template <typename IoT, typename BcT>
__host__ __device__ constexpr int bwd_warp_smem() {
    return 2 * (int)sizeof(BwdStage<IoT, BcT>) + kBwdSteps * 32 * (int)sizeof(float) +
           kEntRows * (kNPad / 4) * 32 * (int)sizeof(float4) +
           32 * kRedStride * (int)sizeof(float);
}

template <int kVecs>
__device__ __forceinline__ void unpack_rows(const uint4 (&r)[kVecs], float (&v)[kBwdSteps]) {
    if constexpr (kVecs == 1) {
        unpack16(r[0], v);
    } else {
        float a[4], b[4];
        unpack16(r[0], a);
        unpack16(r[1], b);
#pragma unroll
        for (int i = 0; i < 4; ++i) { v[i] = a[i]; v[4 + i] = b[i]; }
    }
}

// Column `lane` of a staged (8 steps x 32 channels) tile of a (batch,
// seqlen, dim) tensor: this lane's channel over the block's steps.
template <typename T, int kVecs>
__device__ __forceinline__ void unpack_col(const uint4 (&tile)[32][kVecs], int lane,
                                           float (&v)[kBwdSteps]) {
    const T* t = reinterpret_cast<const T*>(&tile[0][0]);
#pragma unroll
    for (int i = 0; i < kBwdSteps; ++i) v[i] = DType<T>::load(t + i * 32 + lane);
}

__device__ __forceinline__ float sigmoid_f32(float x) {
    return __fdividef(1.0f, 1.0f + ex2_approx(-x * kLog2e));
}

// Abar and Delta as the forward computes them (MUFU ex2 and the lg2 softplus
// for bf16 inputs, the unbiased forms for fp32), so that the recomputed states
// follow the forward's arithmetic.
template <bool kExact>
__device__ __forceinline__ float2 bwd_exp2x2(float2 x) {
    if constexpr (kExact) return exp2_near_one_exact2(x);
    return make_float2(ex2_approx(x.x), ex2_approx(x.y));
}

// dg/dA / Delta^2 = (x e^x - expm1(x)) / x^2 for x = Delta A, as its series
// sum_k x^k (k + 1) / (k + 2)! written in x2 = x log2(e) (coefficients
// ln2^k (k + 1) / (k + 2)!), nine terms: truncation below 2e-9 relative for
// |x2| < kDgdaSmall.  Beyond it the closed form Delta (Abar - phi) / A loses
// at most a few units of 1e-6 to cancellation.
constexpr float kDgdaSmall = 0.75f;

__device__ __forceinline__ float2 zoh_dgda_series2(float2 x2) {
    constexpr float c[9] = {0.5f, 0.23104906018664842f, 0.060056626739775174f,
                            0.011100821732964315f, 0.0016030215179380792f,
                            0.0001904794020918349f, 1.925441299172701e-05f,
                            1.694748200451093e-06f, 1.3215486790144306e-07f};
    float2 r = make_float2(c[8], c[8]);
#pragma unroll
    for (int k = 7; k >= 0; --k) r = __ffma2_rn(x2, r, make_float2(c[k], c[k]));
    return r;
}

template <typename IoT, typename BcT, bool kHasZ, bool kZoh, bool kBld>
__global__ void __launch_bounds__(kBwdWarps * 32)
    selective_scan_bwd_kernel(const __grid_constant__ BwdParams p) {
    constexpr bool kExact = sizeof(IoT) == 4;
    using Stage = BwdStage<IoT, BcT>;
    constexpr int kIoVecs = Stage::kIoRow / 16, kBcVecs = Stage::kBcRow / 16;
    extern __shared__ __align__(16) uint8_t bwd_smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    uint8_t* wbase = bwd_smem + warp * bwd_warp_smem<IoT, BcT>();
    Stage* stages = reinterpret_cast<Stage*>(wbase);
    float (*bcf)[32] = reinterpret_cast<float (*)[32]>(wbase + 2 * sizeof(Stage));
    float4 (*ent)[kNPad / 4][32] = reinterpret_cast<float4 (*)[kNPad / 4][32]>(
        wbase + 2 * sizeof(Stage) + kBwdSteps * 32 * sizeof(float));
    float (*rbuf)[kRedStride] = reinterpret_cast<float (*)[kRedStride]>(
        wbase + 2 * sizeof(Stage) + kBwdSteps * 32 * sizeof(float) +
        kEntRows * (kNPad / 4) * 32 * sizeof(float4));
    // The partial this lane sums in the reduction of a quarter: dB (lanes
    // 0..15) or dC (16..31), step (lane & 15) / 2, entries 2 (lane & 1) + 0, 1.
    const int red_kind = lane >> 4;
    const int red_t = (lane & 15) >> 1;
    const int red_n = (lane & 1) * 2;

    for (;;) {
        unsigned int item = 0;
        if (lane == 0) item = atomicAdd(p.counter, 1u);
        item = __shfl_sync(0xffffffffu, item, 0);
        if ((int64_t)item >= p.items) break;
        const int64_t g = item % p.groups;
        const int64_t kr = item / p.groups;                  // segments done after this one
        const int64_t k = p.nseg - 1 - kr;
        const int64_t b = g / p.groups_per_batch;
        const int64_t d0 = (g % p.groups_per_batch) * 32;
        const int64_t d = d0 + lane;
        const bool valid = d < p.dim;
        const int64_t chain = b * p.dim + (valid ? d : 0);
        const int64_t t_begin = k * p.seg_len;
        const int64_t t_end = min(t_begin + p.seg_len, p.seqlen);

        // per-entry values of the lane's channel, one float4 per quarter
#pragma unroll
        for (int q = 0; q < kNPad / 4; ++q) {
            float a2v[4], iva[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int n = 4 * q + i;
                const bool on = valid && n < p.dstate;
                const float a = on ? p.A[d * p.dstate + n] : 0.0f;
                a2v[i] = a * kLog2e;
                iva[i] = on ? 1.0f / a : 0.0f;       // 1 / A_n, as the forward holds it
            }
            ent[kEntA2][q][lane] = make_float4(a2v[0], a2v[1], a2v[2], a2v[3]);
            if (kZoh) ent[kEntInvA][q][lane] = make_float4(iva[0], iva[1], iva[2], iva[3]);
            ent[kEntDA][q][lane] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
        const float bias = (valid && p.delta_bias != nullptr) ? p.delta_bias[d] : 0.0f;
        const float Dd = (valid && p.D != nullptr) ? p.D[d] : 0.0f;

        if (kr == 0) {
#pragma unroll
            for (int q = 0; q < kNPad / 4; ++q) {
                float l[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int n = 4 * q + i;
                    l[i] = (valid && p.dlast != nullptr && n < p.dstate)
                               ? p.dlast[chain * p.dstate + n] : 0.0f;
                }
                ent[kEntLam][q][lane] = make_float4(l[0], l[1], l[2], l[3]);
            }
        } else {
            bool ok = true;
            if (lane == 0) {
                ok = false;
                for (uint32_t i = 0; i < p.flag_poll_limit; ++i) {
                    if (ld_acquire_gpu(p.flags + g) >= (unsigned int)kr) {
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
            float2 c2[kNPad / 2];
            load16(p.carry + chain * kNPad, c2);
#pragma unroll
            for (int q = 0; q < kNPad / 4; ++q)
                ent[kEntLam][q][lane] = valid ? make_float4(c2[2 * q].x, c2[2 * q].y,
                                                            c2[2 * q + 1].x, c2[2 * q + 1].y)
                                              : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
        float dD_acc = 0.0f, dbias_acc = 0.0f;

        // This lane's channel of u, delta, z, dout and the gradients: step t at
        // row[t] ((batch, dim, seqlen)), or at row[t * dim] ((batch, seqlen, dim)).
        const int64_t io_base = kBld ? b * p.seqlen * p.dim + (valid ? d : 0) : chain * p.seqlen;
        const int64_t io_step = kBld ? p.dim : 1;
        const IoT* urow = static_cast<const IoT*>(p.u) + io_base;
        const IoT* drow = static_cast<const IoT*>(p.delta) + io_base;
        const IoT* zrow = kHasZ ? static_cast<const IoT*>(p.z) + io_base : nullptr;
        const IoT* grow = static_cast<const IoT*>(p.dout) + io_base;
        const bool vec = !kBld && p.vec_ok && (p.seqlen * (int64_t)sizeof(IoT)) % 16 == 0 && valid;
        const int nblk = (int)((t_end - t_begin + kBwdSteps - 1) / kBwdSteps);
        const int nbc = lane & 15;
        const BcT* bcrow = static_cast<const BcT*>(lane < 16 ? p.B : p.C) +
                           (b * p.dstate + (nbc < p.dstate ? nbc : 0)) * p.seqlen;
        // Blocks are staged one ahead by cp.async when every row is 16-byte
        // aligned (with (batch, seqlen, dim): a row of channels, and the
        // group's 32 channels all present); a block shorter than 8 steps (the
        // sequence's last) is read directly.
        const bool pipe = p.vec_ok && p.bc_vec &&
                          (kBld ? (p.dim * (int64_t)sizeof(IoT)) % 16 == 0 && d0 + 32 <= p.dim
                                : (p.seqlen * (int64_t)sizeof(IoT)) % 16 == 0);
        auto issue = [&](int jj) {
            const int64_t tt = t_begin + (int64_t)jj * kBwdSteps;
            if (pipe && t_end - tt >= kBwdSteps) {
                Stage& S = stages[jj & 1];
                if constexpr (kBld) {
                    // each tensor's (8 steps x 32 channels) tile, row r = step:
                    // lane l copies the 16-byte chunk(s) (l & 3) of row l >> 2
                    constexpr int kChunks = (int)sizeof(IoT) / 2;   // 1 (bf16) or 2 (fp32)
                    const int r = lane >> 2;
                    const int64_t roff = (b * p.seqlen + tt + r) * p.dim + d0;
#pragma unroll
                    for (int v = 0; v < kChunks; ++v) {
                        const int ci = (lane & 3) * kChunks + v;
                        const int64_t src = roff + ci * (16 / (int)sizeof(IoT));
                        const int dst = r * 32 * (int)sizeof(IoT) + ci * 16;
                        cp_async16(reinterpret_cast<uint8_t*>(&S.io[0][0][0]) + dst, static_cast<const IoT*>(p.u) + src);
                        cp_async16(reinterpret_cast<uint8_t*>(&S.io[1][0][0]) + dst, static_cast<const IoT*>(p.delta) + src);
                        if (kHasZ) cp_async16(reinterpret_cast<uint8_t*>(&S.io[2][0][0]) + dst, static_cast<const IoT*>(p.z) + src);
                        cp_async16(reinterpret_cast<uint8_t*>(&S.io[3][0][0]) + dst, static_cast<const IoT*>(p.dout) + src);
                    }
                    const float* ckq = p.ckpt + (chain * p.ckpt_tiles + tt / kBwdSteps) * kNPad;
#pragma unroll
                    for (int v = 0; v < 4; ++v) cp_async16(&S.ck[lane][v], ckq + 4 * v);
                } else if (valid) {
#pragma unroll
                    for (int v = 0; v < kIoVecs; ++v) {
                        cp_async16(&S.io[0][lane][v], urow + tt + v * (16 / (int)sizeof(IoT)));
                        cp_async16(&S.io[1][lane][v], drow + tt + v * (16 / (int)sizeof(IoT)));
                        if (kHasZ) cp_async16(&S.io[2][lane][v], zrow + tt + v * (16 / (int)sizeof(IoT)));
                        cp_async16(&S.io[3][lane][v], grow + tt + v * (16 / (int)sizeof(IoT)));
                    }
                    const float* ckq = p.ckpt + (chain * p.ckpt_tiles + tt / kBwdSteps) * kNPad;
#pragma unroll
                    for (int v = 0; v < 4; ++v) cp_async16(&S.ck[lane][v], ckq + 4 * v);
                }
                if (nbc < p.dstate) {
#pragma unroll
                    for (int v = 0; v < kBcVecs; ++v)
                        cp_async16(&S.bc[lane][v], bcrow + tt + v * (16 / (int)sizeof(BcT)));
                }
            }
            cp_async_commit();                   // possibly empty: one group per block
        };
        issue(nblk - 1);

        for (int j = nblk - 1; j >= 0; --j) {
            const int64_t t0 = t_begin + (int64_t)j * kBwdSteps;
            const int ns = (int)min((int64_t)kBwdSteps, t_end - t0);
            if (j > 0) {
                issue(j - 1);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            // A lane reads a column of a (batch, seqlen, dim) tile whose rows
            // other lanes copied: their copies must have landed.
            if constexpr (kBld) __syncwarp();
            const bool staged = pipe && ns == kBwdSteps;
            const Stage& S = stages[j & 1];
            const float4* ck4 = reinterpret_cast<const float4*>(
                p.ckpt + (chain * p.ckpt_tiles + t0 / kBwdSteps) * kNPad);
            // ---- inputs of this block: the lane's own channel, and the B/C table.
            // Steps past the end of a short block read as zero.
            float uu[kBwdSteps], dt[kBwdSteps], dy[kBwdSteps], aux[kBwdSteps];
            if (valid && staged) {
                if constexpr (kBld) {
                    unpack_col<IoT, kIoVecs>(S.io[0], lane, uu);
                    unpack_col<IoT, kIoVecs>(S.io[1], lane, dt);
                    unpack_col<IoT, kIoVecs>(S.io[3], lane, dy);
                    if (kHasZ) unpack_col<IoT, kIoVecs>(S.io[2], lane, aux);
                } else {
                    unpack_rows<kIoVecs>(S.io[0][lane], uu);
                    unpack_rows<kIoVecs>(S.io[1][lane], dt);   // delta, turned into Delta below
                    unpack_rows<kIoVecs>(S.io[3][lane], dy);   // dout, turned into dy below
                    if (kHasZ) unpack_rows<kIoVecs>(S.io[2][lane], aux);
                }
            } else if (valid) {
                if constexpr (kBld) {
                    load_block_strided(urow, t0, ns, io_step, uu);
                    load_block_strided(drow, t0, ns, io_step, dt);
                    load_block_strided(grow, t0, ns, io_step, dy);
                    if (kHasZ) load_block_strided(zrow, t0, ns, io_step, aux);
                } else {
                    load_block(urow, t0, ns, vec, uu);
                    load_block(drow, t0, ns, vec, dt);
                    load_block(grow, t0, ns, vec, dy);
                    if (kHasZ) load_block(zrow, t0, ns, vec, aux);
                }
            } else {
#pragma unroll
                for (int i = 0; i < kBwdSteps; ++i) uu[i] = dt[i] = dy[i] = aux[i] = 0.0f;
            }
            {
                float row[kBwdSteps];
                if (nbc >= p.dstate) {
#pragma unroll
                    for (int i = 0; i < kBwdSteps; ++i) row[i] = 0.0f;
                } else if (staged) {
                    unpack_rows<kBcVecs>(S.bc[lane], row);
                } else {
                    load_block(bcrow, t0, ns, p.bc_vec != 0, row);
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < kBwdSteps; ++i) bcf[i][lane] = row[i];
                __syncwarp();
            }
            // Delta, dy and the gate factor.  Delta is zero past the block's
            // end, so that those steps leave the state and lambda as they are
            // (Abar = 1, no input).
#pragma unroll
            for (int i = 0; i < kBwdSteps; ++i) {
                const float s = dt[i] + bias;
                const float dlt = p.softplus ? (kExact ? softplus_f32(s) : softplus_lg2(s)) : s;
                dt[i] = (valid && i < ns) ? dlt : 0.0f;
                if (kHasZ) {
                    const float zv = aux[i];
                    const float sg = sigmoid_f32(zv);
                    const float gd = dy[i];
                    dy[i] = gd * zv * sg;                              // dout * silu(z)
                    aux[i] = gd * sg * fmaf(zv, 1.0f - sg, 1.0f);      // dout * silu'(z)
                }
            }
            // Sums over the 16 entries, kept as pairs: y (the forward's readout),
            // the Delta adjoint and sum_n lambda B (phi B for the zero-order hold).
            float2 y2[kBwdSteps], dd2[kBwdSteps], db2[kBwdSteps];
#pragma unroll
            for (int i = 0; i < kBwdSteps; ++i)
                y2[i] = dd2[i] = db2[i] = make_float2(0.0f, 0.0f);

            // One state quarter per pass (the loop body is emitted once).
#pragma unroll 1
            for (int q = 0; q < kNPad / 4; ++q) {
                const int n0 = 4 * q;
                // The four entries run as two fp32x2 pairs (packed FMA/FMUL,
                // rounding identical to the scalar forms).
                const float4 a4 = ent[kEntA2][q][lane];
                const float2 a2p[2] = {make_float2(a4.x, a4.y), make_float2(a4.z, a4.w)};
                const float2 a2l[2] = {__fmul2_rn(a2p[0], make_float2(kLn2, kLn2)),
                                       __fmul2_rn(a2p[1], make_float2(kLn2, kLn2))};
                float2 iv[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
                if (kZoh) {
                    const float4 v = ent[kEntInvA][q][lane];
                    iv[0] = make_float2(v.x, v.y);
                    iv[1] = make_float2(v.z, v.w);
                }
                // phi(Delta A) of the zero-order hold, as the forward forms it:
                // its series near 0, else (Abar - 1) / (Delta A).
                auto zoh_phi2 = [&](float2 x2, float2 ab, float rdt, int pr) -> float2 {
                    const float2 big = __fmul2_rn(__fadd2_rn(ab, make_float2(-1.0f, -1.0f)),
                                                  __fmul2_rn(make_float2(rdt, rdt), iv[pr]));
                    const float2 ser = zoh_phi_series2(x2);
                    return make_float2(fabsf(x2.x) < kZohSmall ? ser.x : big.x,
                                       fabsf(x2.y) < kZohSmall ? ser.y : big.y);
                };
                float4 c4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (staged) {
                    if (valid) {
                        const uint4 r = S.ck[lane][q];
                        c4 = make_float4(__uint_as_float(r.x), __uint_as_float(r.y),
                                         __uint_as_float(r.z), __uint_as_float(r.w));
                    }
                } else if (valid) {
                    c4 = __ldcg(ck4 + q);
                }
                // forward: the block's 8 states of entries n0..n0+3, and Abar
                // (kept for the way back)
                float2 hq[kBwdSteps][2], abq[kBwdSteps][2];
                float2 h2[2] = {make_float2(c4.x, c4.y), make_float2(c4.z, c4.w)};
#pragma unroll
                for (int t = 0; t < kBwdSteps; ++t) {
                    const float4 Bq = *reinterpret_cast<const float4*>(&bcf[t][n0]);
                    const float4 Cq = *reinterpret_cast<const float4*>(&bcf[t][16 + n0]);
                    const float2 bq[2] = {make_float2(Bq.x, Bq.y), make_float2(Bq.z, Bq.w)};
                    const float2 cq[2] = {make_float2(Cq.x, Cq.y), make_float2(Cq.z, Cq.w)};
                    const float du = dt[t] * uu[t];
                    const float2 dt2 = make_float2(dt[t], dt[t]), du2 = make_float2(du, du);
                    const float rdt = kZoh ? __fdividef(1.0f, dt[t]) : 0.0f;
#pragma unroll
                    for (int pr = 0; pr < 2; ++pr) {
                        const float2 x2 = __fmul2_rn(dt2, a2p[pr]);
                        const float2 ab = bwd_exp2x2<kExact>(x2);
                        float2 in = __fmul2_rn(du2, bq[pr]);
                        if (kZoh) in = __fmul2_rn(in, zoh_phi2(x2, ab, rdt, pr));
                        h2[pr] = __ffma2_rn(ab, h2[pr], in);
                        hq[t][pr] = h2[pr];
                        abq[t][pr] = ab;
                        y2[t] = __ffma2_rn(cq[pr], h2[pr], y2[t]);
                    }
                }
                // reverse: the adjoint of entries n0..n0+3 over the block
                const float4 l4 = ent[kEntLam][q][lane];
                const float4 g4 = ent[kEntDA][q][lane];
                float2 l2[2] = {make_float2(l4.x, l4.y), make_float2(l4.z, l4.w)};
                float2 dA2[2] = {make_float2(g4.x, g4.y), make_float2(g4.z, g4.w)};
#pragma unroll
                for (int t = kBwdSteps - 1; t >= 0; --t) {
                    const float4 Bq = *reinterpret_cast<const float4*>(&bcf[t][n0]);
                    const float4 Cq = *reinterpret_cast<const float4*>(&bcf[t][16 + n0]);
                    const float2 bq[2] = {make_float2(Bq.x, Bq.y), make_float2(Bq.z, Bq.w)};
                    const float2 cq[2] = {make_float2(Cq.x, Cq.y), make_float2(Cq.z, Cq.w)};
                    const float du = dt[t] * uu[t];
                    const float2 dt2 = make_float2(dt[t], dt[t]), du2 = make_float2(du, du);
                    const float2 ndu2 = make_float2(-du, -du), dy2 = make_float2(dy[t], dy[t]);
                    const float2 uu2 = make_float2(uu[t], uu[t]);
                    const float rdt = kZoh ? __fdividef(1.0f, dt[t]) : 0.0f;
                    float2 rb[2], rc[2];
#pragma unroll
                    for (int pr = 0; pr < 2; ++pr) {
                        l2[pr] = __ffma2_rn(cq[pr], dy2, l2[pr]);                    // lambda_t
                        const float2 ab = abq[t][pr];
                        rc[pr] = __fmul2_rn(dy2, hq[t][pr]);                          // dC
                        if (!kZoh) {
                            const float2 abh = __ffma2_rn(ndu2, bq[pr], hq[t][pr]);  // Abar_t h_t-1
                            rb[pr] = __fmul2_rn(l2[pr], du2);                         // dB
                            dd2[t] = __ffma2_rn(l2[pr], __ffma2_rn(a2l[pr], abh, __fmul2_rn(bq[pr], uu2)), dd2[t]);
                            db2[t] = __ffma2_rn(l2[pr], bq[pr], db2[t]);
                            dA2[pr] = __ffma2_rn(__fmul2_rn(l2[pr], dt2), abh, dA2[pr]);
                        } else {
                            const float2 x2 = __fmul2_rn(dt2, a2p[pr]);
                            const float2 phi = zoh_phi2(x2, ab, rdt, pr);
                            const float2 bu = __fmul2_rn(bq[pr], uu2);                // B u
                            const float2 in = __fmul2_rn(__fmul2_rn(du2, bq[pr]), phi);
                            const float2 abh = __fadd2_rn(hq[t][pr], make_float2(-in.x, -in.y));
                            rb[pr] = __fmul2_rn(l2[pr], __fmul2_rn(du2, phi));        // dB
                            dd2[t] = __ffma2_rn(l2[pr], __ffma2_rn(a2l[pr], abh, __fmul2_rn(ab, bu)), dd2[t]);
                            db2[t] = __ffma2_rn(l2[pr], __fmul2_rn(phi, bq[pr]), db2[t]);
                            // dg/dA: Delta^2 times its series near 0, else Delta (Abar - phi) / A
                            const float2 ser = __fmul2_rn(__fmul2_rn(dt2, dt2), zoh_dgda_series2(x2));
                            const float2 big = __fmul2_rn(dt2, __fmul2_rn(__fadd2_rn(ab, make_float2(-phi.x, -phi.y)), iv[pr]));
                            const float2 dgda = make_float2(fabsf(x2.x) < kDgdaSmall ? ser.x : big.x,
                                                            fabsf(x2.y) < kDgdaSmall ? ser.y : big.y);
                            dA2[pr] = __ffma2_rn(l2[pr], __ffma2_rn(dt2, abh, __fmul2_rn(dgda, bu)), dA2[pr]);
                        }
                        l2[pr] = __fmul2_rn(l2[pr], ab);                              // to h_t-1
                    }
                    *reinterpret_cast<float4*>(&rbuf[lane][4 * t]) =
                        make_float4(rb[0].x, rb[0].y, rb[1].x, rb[1].y);
                    *reinterpret_cast<float4*>(&rbuf[lane][4 * kBwdSteps + 4 * t]) =
                        make_float4(rc[0].x, rc[0].y, rc[1].x, rc[1].y);
                }
                ent[kEntLam][q][lane] = make_float4(l2[0].x, l2[0].y, l2[1].x, l2[1].y);
                ent[kEntDA][q][lane] = make_float4(dA2[0].x, dA2[0].y, dA2[1].x, dA2[1].y);
                // dB and dC sum over the warp's 32 channels: each lane adds one
                // pair of the 64 partials over the 32 rows and adds the pair to
                // global memory.
                __syncwarp();
                float2 acc[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int src = 0; src < 32; ++src)
                    acc[src & 3] = __fadd2_rn(acc[src & 3],
                                              *reinterpret_cast<const float2*>(&rbuf[src][2 * lane]));
                const float2 tot = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
                __syncwarp();
                const int n = n0 + red_n;
                if (red_t < ns && n < p.dstate) {
                    float* dst = (red_kind ? p.dC : p.dB) + (b * p.dstate + n) * p.seqlen + t0 + red_t;
                    atomicAdd(dst, tot.x);
                    if (n + 1 < p.dstate) atomicAdd(dst + p.seqlen, tot.y);
                }
            }
            // per-step outputs of the block; the softplus derivative
            // sigmoid(delta + bias) from delta read again
            float sp[kBwdSteps];
            if (p.softplus) {
                if (valid && staged) {
                    if constexpr (kBld) unpack_col<IoT, kIoVecs>(S.io[1], lane, sp);
                    else unpack_rows<kIoVecs>(S.io[1][lane], sp);
                } else if (valid) {
                    if constexpr (kBld) load_block_strided(drow, t0, ns, io_step, sp);
                    else load_block(drow, t0, ns, vec, sp);
                } else {
#pragma unroll
                    for (int i = 0; i < kBwdSteps; ++i) sp[i] = 0.0f;
                }
#pragma unroll
                for (int i = 0; i < kBwdSteps; ++i) sp[i] = sigmoid_f32(sp[i] + bias);
            } else {
#pragma unroll
                for (int i = 0; i < kBwdSteps; ++i) sp[i] = 1.0f;
            }
            float o_du[kBwdSteps], o_dd[kBwdSteps], o_dz[kBwdSteps];
#pragma unroll
            for (int t = 0; t < kBwdSteps; ++t) {
                const bool in = t < ns;
                o_du[t] = fmaf(Dd, dy[t], dt[t] * (db2[t].x + db2[t].y));
                const float ds = (dd2[t].x + dd2[t].y) * sp[t];
                o_dd[t] = ds;
                if (in) {
                    dbias_acc += ds;
                    dD_acc = fmaf(dy[t], uu[t], dD_acc);
                }
                o_dz[t] = kHasZ ? aux[t] * fmaf(Dd, uu[t], y2[t].x + y2[t].y) : 0.0f;
            }
            __syncwarp();
            if (valid) {
                if constexpr (kBld) {   // 32 lanes write 32 consecutive channels of a step
                    store_block_strided(static_cast<IoT*>(p.du) + io_base, t0, ns, io_step, o_du);
                    store_block_strided(static_cast<IoT*>(p.ddelta) + io_base, t0, ns, io_step, o_dd);
                    if (kHasZ && p.dz != nullptr)
                        store_block_strided(static_cast<IoT*>(p.dz) + io_base, t0, ns, io_step, o_dz);
                } else {
                    store_block(static_cast<IoT*>(p.du) + chain * p.seqlen, t0, ns, vec, o_du);
                    store_block(static_cast<IoT*>(p.ddelta) + chain * p.seqlen, t0, ns, vec, o_dd);
                    if (kHasZ && p.dz != nullptr)
                        store_block(static_cast<IoT*>(p.dz) + chain * p.seqlen, t0, ns, vec, o_dz);
                }
            }
        }

        // hand lambda to the earlier segment, or it is the start state's gradient
        float lam[kNPad], dA_acc[kNPad];
#pragma unroll
        for (int q = 0; q < kNPad / 4; ++q) {
            const float4 l4 = ent[kEntLam][q][lane];
            const float4 g4 = ent[kEntDA][q][lane];
            lam[4 * q] = l4.x; lam[4 * q + 1] = l4.y; lam[4 * q + 2] = l4.z; lam[4 * q + 3] = l4.w;
            dA_acc[4 * q] = g4.x; dA_acc[4 * q + 1] = g4.y; dA_acc[4 * q + 2] = g4.z; dA_acc[4 * q + 3] = g4.w;
        }
        if (k > 0) {
            float2 c2[kNPad / 2];
#pragma unroll
            for (int i = 0; i < kNPad / 2; ++i) c2[i] = make_float2(lam[2 * i], lam[2 * i + 1]);
            if (valid) store16(p.carry + chain * kNPad, c2);
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_gpu(p.flags + g, (unsigned int)(kr + 1));
        } else if (valid && p.dh0 != nullptr) {
#pragma unroll
            for (int n = 0; n < kNPad; ++n)
                if (n < p.dstate) p.dh0[chain * p.dstate + n] = lam[n];
        }
        if (valid) {
#pragma unroll
            for (int n = 0; n < kNPad; ++n)
                if (n < p.dstate) atomicAdd(p.dA + d * p.dstate + n, dA_acc[n]);
            if (p.dD != nullptr) atomicAdd(p.dD + d, dD_acc);
            if (p.dbias != nullptr) atomicAdd(p.dbias + d, dbias_acc);
        }
    }
}

}  // namespace mamba
