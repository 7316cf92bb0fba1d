// Mamba-2 layer (scalar A per head) on the 5th-generation tensor cores.
//
// "Mamba 与状态空间模型", section "Mamba-2：两种算法": with A a scalar times the
// identity, the layer is one lower-triangular matrix M applied to the input,
// M_ij = C_i . B_j x (all the decay between steps j and i) x Delta_j.  The
// sequence is cut into chunks: inside a chunk M is applied as dense products
// (the tensor cores' work), and only the (headdim x dstate) state crosses
// from one chunk to the next.
//
// One CTA of 128 threads owns one (batch, head) chain and walks its chunks
// of Q = 128 tokens in order.  Per chunk, with c_i the running log2-decay
// (c_i = log2(e) A_h sum_{r<=i} Delta_r inside the chunk) and H the state
// entering the chunk (fp32, one TMEM lane / thread per state index n):
//
//   G     = C B^T                       (Q x Q,  K = dstate)        MMA 1
//   Yoff  = C H^T                       (Q x P,  K = dstate)        MMA 3
//   S^T   = B^T Xw, Xw_j = 2^(c_Q - c_j) Delta_j x_j   (N x P, K = Q) MMA 4
//   Gm_ij = G_ij 2^(c_i - c_j) Delta_j  for j <= i, else 0  (CUDA cores)
//   Ydiag = Gm X                        (Q x P,  K = Q)             MMA 2
//   y_i   = Ydiag_i + 2^(c_i) Yoff_i + D_h x_i,  out = y silu(z)
//   H     = 2^(c_Q) H + S               (fp32, in registers)
//
// Operands are bf16 in shared memory in the no-swizzle canonical layout
// ("core matrices" of 8 rows x 16 bytes); the products accumulate in fp32 in
// tensor memory and are read back with tcgen05.ld.  One elected thread
// issues the tcgen05.mma instructions and commits them to an mbarrier that
// the CTA waits on (bounded).  Delta_j enters only through
// e_j = c_j - log2(Delta_j), so that 2^(c_i - e_j) = 2^(c_i - c_j) Delta_j
// and padded tokens (Delta = 0, e = +inf) drop out by themselves.
#pragma once

#include "ssm_device.cuh"

namespace mamba {

constexpr int kSsdP = 64;          // head dimension
constexpr int kSsdN = 128;         // state size
constexpr int kSsdQ = 128;         // chunk length
constexpr int kSsdThreads = 128;   // one thread per TMEM lane
constexpr int kSsdTmemCols = 256;  // G [0,128) (then Ydiag [0,64)), Yoff [128,192), S [192,256)

// Shared-memory map (bytes).  sC holds C and later Gm; all operand tiles use
// offset(row, k) = (k / 8) * 2048 + row * 16 + (k % 8) * 2 for 128 rows.
constexpr int kSsdOffC = 0;          // 128 x 128 bf16: C (rows i, k = n), then Gm (rows i, k = j)
constexpr int kSsdOffB = 32768;      // 128 x 128 bf16: B (rows j, k = n)
constexpr int kSsdOffX = 65536;      // 128 x 64 bf16: x (rows j, k = p)
constexpr int kSsdOffXw = 81920;     // 128 x 64 bf16: Xw (rows j, k = p)
constexpr int kSsdOffH = 98304;      // 128 x 64 bf16: H (rows n, k = p)
constexpr int kSsdOffE = 114688;     // 128 fp32: e_j = c_j - log2(Delta_j)
constexpr int kSsdOffMisc = 115200;  // two mbarriers (+8, +16), the TMEM address (+24)
constexpr int kSsdSmemBytes = 115232;

struct SsdParams {
    const __nv_bfloat16* x;      // (batch, L, nheads, 64)
    const __nv_bfloat16* dt;     // (batch, L, nheads)
    const float* A;              // (nheads)
    const __nv_bfloat16* B;      // (batch, L, ngroups, 128)
    const __nv_bfloat16* C;      // (batch, L, ngroups, 128)
    const float* D;              // (nheads) or null
    const __nv_bfloat16* z;      // like x, or null
    const float* dt_bias;        // (nheads) or null
    const float* h0;             // (batch, nheads, 64, 128) or null
    __nv_bfloat16* out;          // like x
    float* hT;                   // (batch, nheads, 64, 128) or null
    int64_t seqlen;
    int nheads, ngroups, softplus;
};

// ---------------------------------------------------------------- tcgen05 PTX

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B,
// M x N tile, each operand K-major (false) or MN-major (true).
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor, no swizzle: start address, leading-byte
// offset (between the two 8-wide core-matrix columns along K for K-major,
// between 8-deep K blocks for MN-major), stride-byte offset (between 8-row
// blocks along M/N), version 1.
__device__ __forceinline__ uint64_t umma_sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05.mma this thread issued has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(slot), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane; the wait for the
// load is in the same statement, so no use of the values can precede it.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(r[k]);
}

__device__ __forceinline__ void cp_async_wait_all_copies() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// 16-byte cp.async that fills zeros instead of reading when `valid` is false.
__device__ __forceinline__ void cp_async16_or_zero(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(valid ? 16 : 0)
                 : "memory");
}


// The state H of this thread's row n as bf16 into sH: offset (p / 8) * 2048 + n * 16.
__device__ __forceinline__ void ssd_store_state(unsigned char* smem, int n, const float (&H)[kSsdP]) {
#pragma unroll
    for (int q = 0; q < kSsdP / 8; ++q) {
        float f[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) f[k] = H[q * 8 + k];
        *reinterpret_cast<uint4*>(smem + kSsdOffH + q * 2048 + n * 16) = pack16(f);
    }
}

// Wait for one commit of the tensor-core work; true on every thread if any
// thread's bounded wait gave up.
__device__ __forceinline__ bool ssd_wait_failed(uint32_t bar, uint32_t parity) {
    const bool ok = mbar_wait_bounded(bar, parity);
    const bool failed = __syncthreads_or(!ok) != 0;
    tc_fence_after();
    return failed;
}

__global__ void __launch_bounds__(kSsdThreads, 2) ssd_chunk_scan_kernel(const SsdParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chain = blockIdx.x;                           // b * nheads + h
    const int h = chain % p.nheads;
    const int64_t b = chain / p.nheads;
    const int g = h / (p.nheads / p.ngroups);
    const int64_t L = p.seqlen;
    const uint32_t s0 = smem_u32(smem);
    float* sE = reinterpret_cast<float*>(smem + kSsdOffE);
    const uint32_t bar1 = s0 + kSsdOffMisc + 8, bar2 = s0 + kSsdOffMisc + 16;
    const uint32_t* tslot = reinterpret_cast<const uint32_t*>(smem + kSsdOffMisc + 24);

    if (warp == 0) tmem_alloc(s0 + kSsdOffMisc + 24, kSsdTmemCols);
    if (tid == 0) {
        mbar_init(bar1, 1);
        mbar_init(bar2, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t tlane = tmem + ((uint32_t)(warp * 32) << 16);   // this warp's 32 lanes

    const float A2 = p.A[h] * kLog2e;
    const float Dh = p.D ? p.D[h] : 0.0f;
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.0f;

    // Thread n holds row n of the state: H[p] = state[p][n], in fp32.
    float H[kSsdP];
    const size_t hoff = (size_t)chain * kSsdP * kSsdN + tid;
#pragma unroll
    for (int q = 0; q < kSsdP; ++q) H[q] = p.h0 ? p.h0[hoff + (size_t)q * kSsdN] : 0.0f;
    ssd_store_state(smem, tid, H);

    const int64_t xs = (int64_t)p.nheads * kSsdP;   // token stride of x, z, out
    const int64_t bcs = (int64_t)p.ngroups * kSsdN; // token stride of B, C
    const int64_t nchunks = (L + kSsdQ - 1) / kSsdQ;
    bool failed = false;

    for (int64_t c = 0; c < nchunks; ++c) {
        const int64_t l0 = c * kSsdQ;
        const int valid = (int)(L - l0 < kSsdQ ? L - l0 : kSsdQ);
        const uint32_t parity = (uint32_t)(c & 1);

        // ---- operands: C, B (128 x 128) and x (128 x 64) by cp.async, zero rows
        // past the end.  A warp copies 8 rows x 4 pieces of 16 bytes per step:
        // 64 contiguous bytes of each row, four 128-byte runs of shared memory.
        const __nv_bfloat16* Cg = p.C + ((b * L + l0) * p.ngroups + g) * kSsdN;
        const __nv_bfloat16* Bg = p.B + ((b * L + l0) * p.ngroups + g) * kSsdN;
        const __nv_bfloat16* Xg = p.x + ((b * L + l0) * p.nheads + h) * kSsdP;
#pragma unroll
        for (int it = 0; it < 16; ++it) {
            const int q = tid + kSsdThreads * it;
            const int r = (((q >> 5) & 15) << 3) | (q & 7);
            const int kb = ((q >> 9) << 2) | ((q >> 3) & 3);
            const uint32_t off = (uint32_t)(kb * 2048 + r * 16);
            const bool ok = r < valid;
            const int64_t src = ok ? (int64_t)r * bcs + kb * 8 : 0;
            cp_async16_or_zero(s0 + kSsdOffC + off, Cg + src, ok);
            cp_async16_or_zero(s0 + kSsdOffB + off, Bg + src, ok);
        }
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int q = tid + kSsdThreads * it;
            const int r = (((q >> 5) & 15) << 3) | (q & 7);
            const int pb = ((q >> 9) << 2) | ((q >> 3) & 3);
            const bool ok = r < valid;
            cp_async16_or_zero(s0 + kSsdOffX + (uint32_t)(pb * 2048 + r * 16),
                               Xg + (ok ? (int64_t)r * xs + pb * 8 : 0), ok);
        }

        // ---- Delta, the running log2-decay c_i and e_i = c_i - log2(Delta_i).
        float delta = 0.0f;
        if (tid < valid) {
            const float s = __bfloat162float(p.dt[(b * L + l0 + tid) * p.nheads + h]) + bias;
            delta = p.softplus ? softplus_f32(s) : s;
        }
        float a = delta * A2;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, a, o);
            if (lane >= o) a += v;
        }
        float* sTot = reinterpret_cast<float*>(smem + kSsdOffXw);   // Xw is free until below
        if (lane == 31) sTot[warp] = a;
        __syncthreads();
        float pre = 0.0f;
        for (int w = 0; w < warp; ++w) pre += sTot[w];
        const float ci = a + pre;
        const float cQ = (sTot[0] + sTot[1]) + (sTot[2] + sTot[3]);
        sE[tid] = ci - lg2_approx(delta);   // +inf for Delta = 0
        cp_async_wait_all_copies();
        __syncthreads();

        // ---- Xw_j = 2^(c_Q - e_j) x_j = 2^(c_Q - c_j) Delta_j x_j (row j = tid).
        {
            const float w = ex2_approx(cQ - sE[tid]);
#pragma unroll
            for (int pb = 0; pb < kSsdP / 8; ++pb) {
                const uint32_t off = (uint32_t)(pb * 2048 + tid * 16);
                float f[8];
                unpack16(*reinterpret_cast<const uint4*>(smem + kSsdOffX + off), f);
#pragma unroll
                for (int k = 0; k < 8; ++k) f[k] *= w;
                *reinterpret_cast<uint4*>(smem + kSsdOffXw + off) = pack16(f);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- MMA 1 (G = C B^T), 3 (Yoff = C H^T), 4 (S^T = B^T Xw).
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id_g = umma_idesc_bf16(128, 128, false, false);
            constexpr uint32_t id_off = umma_idesc_bf16(128, 64, false, true);
            constexpr uint32_t id_s = umma_idesc_bf16(128, 64, true, true);
#pragma unroll
            for (int k = 0; k < kSsdN / 16; ++k)
                umma_bf16(tmem, umma_sdesc(s0 + kSsdOffC + k * 4096, 2048, 128),
                          umma_sdesc(s0 + kSsdOffB + k * 4096, 2048, 128), id_g, k);
#pragma unroll
            for (int k = 0; k < kSsdN / 16; ++k)
                umma_bf16(tmem + 128, umma_sdesc(s0 + kSsdOffC + k * 4096, 2048, 128),
                          umma_sdesc(s0 + kSsdOffH + k * 256, 128, 2048), id_off, k);
#pragma unroll
            for (int k = 0; k < kSsdQ / 16; ++k)
                umma_bf16(tmem + 192, umma_sdesc(s0 + kSsdOffB + k * 256, 128, 2048),
                          umma_sdesc(s0 + kSsdOffXw + k * 256, 128, 2048), id_s, k);
            umma_commit(bar1);
        }
        if (ssd_wait_failed(bar1, parity)) {
            failed = true;
            break;
        }

        // ---- state: H = 2^(c_Q) H + S (row n = tid), then its bf16 copy for
        // the next chunk's MMA 3.
        {
            const float dq = ex2_approx(cQ);
            float sv[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld32(tlane + 192 + half * 32, sv);
#pragma unroll
                for (int k = 0; k < 32; ++k) H[half * 32 + k] = fmaf(dq, H[half * 32 + k], sv[k]);
            }
            ssd_store_state(smem, tid, H);
        }

        // ---- Gm_ij = G_ij 2^(c_i - e_j) for j <= i (row i = tid), over C's tile.
#pragma unroll
        for (int quarter = 0; quarter < 4; ++quarter) {
            float gv[32];
            tmem_ld32(tlane + quarter * 32, gv);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int j0 = quarter * 32 + q * 8;
                float f[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    f[k] = (j0 + k <= tid) ? gv[q * 8 + k] * ex2_approx(ci - sE[j0 + k]) : 0.0f;
                *reinterpret_cast<uint4*>(smem + kSsdOffC + (j0 / 8) * 2048 + tid * 16) = pack16(f);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA 2: Ydiag = Gm X into columns [0, 64).
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id_y = umma_idesc_bf16(128, 64, false, true);
#pragma unroll
            for (int k = 0; k < kSsdQ / 16; ++k)
                umma_bf16(tmem, umma_sdesc(s0 + kSsdOffC + k * 4096, 2048, 128),
                          umma_sdesc(s0 + kSsdOffX + k * 256, 128, 2048), id_y, k);
            umma_commit(bar2);
        }
        if (ssd_wait_failed(bar2, parity)) {
            failed = true;
            break;
        }

        // ---- y_i = Ydiag_i + 2^(c_i) Yoff_i + D x_i, gated, stored (row i = tid).
        {
            const float sc = ex2_approx(ci);
            const int64_t row = ((b * L + l0 + tid) * p.nheads + h) * kSsdP;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float yd[32], yo[32];
                tmem_ld32(tlane + half * 32, yd);
                tmem_ld32(tlane + 128 + half * 32, yo);
                if (tid < valid) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int p0 = half * 32 + q * 8;
                        float xv[8], f[8];
                        unpack16(*reinterpret_cast<const uint4*>(smem + kSsdOffX + (p0 / 8) * 2048 +
                                                                 tid * 16), xv);
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            f[k] = fmaf(Dh, xv[k], fmaf(sc, yo[q * 8 + k], yd[q * 8 + k]));
                        if (p.z) {
                            float zv[8];
                            unpack16(*reinterpret_cast<const uint4*>(p.z + row + p0), zv);
#pragma unroll
                            for (int k = 0; k < 8; ++k) f[k] *= silu_f32(zv[k]);
                        }
                        *reinterpret_cast<uint4*>(p.out + row + p0) = pack16(f);
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();   // the next chunk rewrites the tiles and the TMEM columns
    }

    if (!failed && p.hT) {
#pragma unroll
        for (int q = 0; q < kSsdP; ++q) p.hT[hoff + (size_t)q * kSsdN] = H[q];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kSsdTmemCols);
    }
    if (failed && tid == 0) record_device_error(MAMBA_ERR_TIMEOUT);
}

}  // namespace mamba
