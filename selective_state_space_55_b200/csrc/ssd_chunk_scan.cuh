// Mamba-2 layer (scalar A per head) on the 5th-generation tensor cores.
//
// "Mamba 与状态空间模型", section "Mamba-2：两种算法": with A a scalar times the
// identity, the layer is one lower-triangular matrix M applied to the input,
// M_ij = C_i . B_j x (all the decay between steps j and i) x Delta_j.  The
// sequence is cut into chunks: inside a chunk M is applied as dense products
// (the tensor cores' work), and only the (headdim x dstate) state crosses
// from one chunk to the next.
//
// One CTA of 256 threads owns one (batch, head) chain and walks its chunks
// of Q = 128 tokens in order; two threads serve each of the 128 TMEM lanes,
// each with half of the head dimension.  Per chunk, with c_i the running
// log2-decay (c_i = log2(e) A_h sum_{r<=i} Delta_r inside the chunk) and H the
// state entering the chunk (fp32 in registers, lane n holds row n of H^T):
//
//   Y     = C H^T                       (Q x P,  K = dstate)        MMA 3
//   S^T   = B^T Xw, Xw_j = 2^(c_Q - c_j) Delta_j x_j   (N x P, K = Q) MMA 4
//   G     = C B^T                       (Q x Q,  K = dstate)        MMA 1
//   Gm_ij = G_ij 2^(c_i - c_j) Delta_j  for j <= i, else 0,
//           plus D_h on the diagonal    (CUDA cores)
//   Y_i  <- 2^(c_i) Y_i                 (CUDA cores, in tensor memory)
//   Y    += Gm X  (intra-chunk part + D_h x)  (Q x P, K = Q)        MMA 2
//   out   = Y silu(z)
//   H     = 2^(c_Q) H + S               (fp32, in registers)
//
// Precision.  The tensor cores multiply bf16 operands.  C, B and x are bf16
// inputs and enter exactly; the three operands the kernel computes (H, Xw
// and Gm) would lose their low bits if rounded to bf16 once, and an output
// that cancels across many terms would then carry an error near 2^-9 times
// the sum of the terms' magnitudes.  Each of them is therefore split as
// v = hi + lo with hi = bf16(v) and lo = bf16(v - hi), and its product is
// issued twice into the same fp32 accumulator; the pair carries v to about
// 2^-17 relative, so the only rounding left at the bf16 level is the one of
// the output itself.
//
// Operands in shared memory are in the tensor cores' 128-byte-swizzle layout
// (1024-byte atoms of 8 rows x 128 bytes).  Gm is formed row by row (thread i
// holds row i) and written straight into tensor memory, from where MMA 2
// reads it as its A operand; this keeps the 2 x 32 KB of Gm out of shared
// memory, which then holds C, B, x and one 32 KB buffer that takes H's hi/lo
// pair for MMA 3 and then Xw's for MMA 4, so two CTAs still fit on an SM.
// One elected thread issues the tcgen05.mma instructions and commits them to
// mbarriers that the CTA waits on (bounded).  Operand tiles arrive by TMA,
// one box per tile, each requested as soon as its buffer is free.  Delta_j
// enters only through e_j = c_j - log2(Delta_j), so that
// 2^(c_i - e_j) = 2^(c_i - c_j) Delta_j and padded tokens (Delta = 0,
// e = +inf) drop out by themselves.
#pragma once

#include "ssm_device.cuh"

namespace mamba {

constexpr int kSsdP = 64;          // head dimension
constexpr int kSsdN = 128;         // state size
constexpr int kSsdQ = 128;         // chunk length
constexpr int kSsdThreads = 256;   // two threads per TMEM lane
constexpr int kSsdTmemCols = 256;
constexpr int kSsdStoreThread = 32;   // issues the output stores (not thread 0, which issues the products)

// Tensor-memory columns (fp32).  G fills [0, 128) until the masked matrix has
// been formed from it; quarter q of Gm (columns j = 32 q .. 32 q + 31, bf16
// pairs) then takes G's own quarter: its lo words in 32 q .. 32 q + 15, its
// hi words in 32 q + 16 .. 32 q + 31.  Y holds C H^T, is scaled in place by
// 2^(c_i) per row, and MMA 2 accumulates Gm X onto it: the output before the
// gate.  S is the chunk's state product.
constexpr uint32_t kTmG = 0;
constexpr uint32_t kTmY = 128;
constexpr uint32_t kTmS = 192;

// Shared-memory map (bytes).  Every operand tile is 128 rows in the
// 128-byte-swizzle layout of the tensor cores: each group of 64 columns
// ("half") is 128 rows of 128 bytes, 8 rows to a 1024-byte atom, and the
// 16-byte chunk c of row r sits at chunk position c ^ (r % 8); halves are
// 16 KB apart.  ssd_sw128 gives the byte offset.
constexpr int kSsdOffC = 0;          // 128 x 128 bf16: C (rows i, k = n)
constexpr int kSsdOffB = 32768;      // 128 x 128 bf16: B (rows j, k = n); once MMA 1 and 4
                                     // are done, its first half takes the gate tile z
constexpr int kSsdOffX = 65536;      // 128 x 64 bf16: x (rows j, k = p); once MMA 2 is
                                     // done, the output tile (rows i, 64 columns p)
constexpr int kSsdOffHX = 81920;     // hi at +0, lo at +16384, each 128 x 64 bf16:
                                     // H (rows n, k = p) for MMA 3, then Xw (rows j, k = p)
constexpr int kSsdOffE = 114688;     // 128 fp32: -e_j, e_j = c_j - log2(Delta_j)
constexpr int kSsdOffBar = 115200;   // 8 mbarriers (see SsdBar)
constexpr int kSsdOffSlot = 115264;  // TMEM base address written by tcgen05.alloc
constexpr int kSsdOffTot = 115280;   // 2 x 4 fp32 warp totals of the decay prefix sum
constexpr int kSsdSmemBytes = 115328;
constexpr uint32_t kSsdLoBytes = 16384;   // offset of the lo half in the HX buffer

// mbarrier indices; each completes at most once per chunk.
enum SsdBar : int {
    kBarC = 0,      // C tile landed
    kBarB = 1,      // B tile landed
    kBarX = 2,      // x tile landed
    kBarZ = 3,      // gate tile landed
    kBarYoff = 4,   // MMA 3 done
    kBarS = 5,      // MMA 4 done
    kBarG = 6,      // MMA 1 done
    kBarYd = 7,     // MMA 2 done
    kSsdBars = 8
};

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

// The same with the 128-byte swizzle (layout type 2).  K-major: rows 128 bytes
// of K, 8-row groups `sbo` = 1024 bytes apart, `lbo` unused (16).  MN-major:
// 64 M/N elements per 128-byte row, K rows in 8-row groups `sbo` apart, the
// next 64 M/N elements `lbo` apart.
__device__ __forceinline__ uint64_t umma_sdesc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return umma_sdesc(addr, lbo, sbo) | (2ull << 61);
}

// Byte offset of 16-byte chunk `chunk` (0..15 over both halves) of row `row`
// in a 128-row swizzled tile.
__device__ __forceinline__ uint32_t ssd_sw128(int row, int chunk) {
    return (uint32_t)((chunk >> 3) * 16384 + (row >> 3) * 1024 + (row & 7) * 128 +
                      (((chunk & 7) ^ (row & 7)) << 4));
}

// D (+)= A B with A and B in shared memory.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D (+)= A B with A in tensor memory (row m in lane m, K-major, two bf16 per
// 32-bit column, the lower K index in the low half) and B in shared memory.
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
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

// 5-D tiled TMA copies of one whole operand tile.  Each map is (64 elements,
// L, column halves, heads or groups, batch) with the box (64, 128, all
// halves, 1, 1) and the 128-byte swizzle, which writes the tile in exactly
// the layout ssd_sw128 describes.  Rows past the end of the sequence are
// filled with zeros on load and dropped on store.
__device__ __forceinline__ void tma_load_tile(uint32_t dst, const CUtensorMap* map, int l0,
                                              int head, int batch, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %2, %4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(l0), "r"(head), "r"(batch), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_store_tile(const CUtensorMap* map, uint32_t src, int l0,
                                               int head, int batch) {
    asm volatile(
        "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %2, %4, %5}], [%1];"
        ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(0), "r"(l0), "r"(head), "r"(batch)
        : "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane from registers.
// Complete (visible to the tensor cores after a fence and barrier) once
// tmem_wait_st returns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
          "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
          "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 1/x on the MUFU pipe (rcp.approx, flush-to-zero); 0 for x = +inf.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// a ~ hi + lo and b likewise: hi = bf16(v), lo = bf16(v - hi), each pair
// packed into one word with a in the low half.  v - hi is exact in fp32
// (hi holds v's leading 8 significant bits), so only lo's own rounding is
// lost: |v - hi - lo| <= 2^-9 |v - hi| <= 2^-17 |v| or so.
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = pack_bf16x2(a, b);
    lo = pack_bf16x2(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xffff0000u));
}

// Eight fp32 values as 16-byte hi and lo chunks.
__device__ __forceinline__ void split16(const float (&f)[8], uint4& hi, uint4& lo) {
    split_bf16x2(f[0], f[1], hi.x, lo.x);
    split_bf16x2(f[2], f[3], hi.y, lo.y);
    split_bf16x2(f[4], f[5], hi.z, lo.z);
    split_bf16x2(f[6], f[7], hi.w, lo.w);
}

// This thread's half of row n of H^T (columns p = 32 hp .. 32 hp + 31) as
// its bf16 hi/lo pair into the HX buffer.
__device__ __forceinline__ void ssd_store_state(unsigned char* smem, int n, int hp,
                                                const float (&H)[kSsdP / 2]) {
#pragma unroll
    for (int q = 0; q < kSsdP / 16; ++q) {
        float f[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) f[k] = H[q * 8 + k];
        uint4 hi, lo;
        split16(f, hi, lo);
        const uint32_t off = ssd_sw128(n, 4 * hp + q);
        *reinterpret_cast<uint4*>(smem + kSsdOffHX + off) = hi;
        *reinterpret_cast<uint4*>(smem + kSsdOffHX + kSsdLoBytes + off) = lo;
    }
}

// One 32-column load of this thread's TMEM lane; valid when it returns.
__device__ __forceinline__ void tmem_ld32(uint32_t ta, float (&a)[32]) {
    uint32_t ra[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(ra[0]), "=r"(ra[1]), "=r"(ra[2]), "=r"(ra[3]), "=r"(ra[4]), "=r"(ra[5]), "=r"(ra[6]), "=r"(ra[7]), "=r"(ra[8]), "=r"(ra[9]), "=r"(ra[10]), "=r"(ra[11]), "=r"(ra[12]), "=r"(ra[13]), "=r"(ra[14]), "=r"(ra[15]), "=r"(ra[16]), "=r"(ra[17]), "=r"(ra[18]), "=r"(ra[19]), "=r"(ra[20]), "=r"(ra[21]), "=r"(ra[22]), "=r"(ra[23]), "=r"(ra[24]), "=r"(ra[25]), "=r"(ra[26]), "=r"(ra[27]), "=r"(ra[28]), "=r"(ra[29]), "=r"(ra[30]), "=r"(ra[31])
        : "r"(ta)
        : "memory");
#pragma unroll
    for (int k = 0; k < 32; ++k) a[k] = __uint_as_float(ra[k]);
}

// 32 consecutive columns of this thread's TMEM lane from fp32 registers.
__device__ __forceinline__ void tmem_st32f(uint32_t taddr, const float (&a)[32]) {
    uint32_t lo[16], hi[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        lo[k] = __float_as_uint(a[k]);
        hi[k] = __float_as_uint(a[16 + k]);
    }
    tmem_st16(taddr, lo);
    tmem_st16(taddr + 16, hi);
}

// Two threads serve each TMEM lane (row) r: threads r and r + 128 ("halves"
// hp = 0, 1), each with half of the head dimension (columns 32 hp .. 32 hp +
// 31 of x, Xw, H, y) and every other column quarter of the masked matrix.
// Tensor memory is accessed by warp w in lanes 32 (w % 4) .. + 31.
__global__ void __launch_bounds__(kSsdThreads, 2)
    ssd_chunk_scan_kernel(const __grid_constant__ SsdParams p,
                          const __grid_constant__ CUtensorMap tm_x,
                          const __grid_constant__ CUtensorMap tm_z,
                          const __grid_constant__ CUtensorMap tm_B,
                          const __grid_constant__ CUtensorMap tm_C,
                          const __grid_constant__ CUtensorMap tm_out) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = tid & (kSsdQ - 1);      // row: token i / j, or state index n
    const int hp = tid >> 7;              // which half of the head dimension
    const int wq = warp & 3;              // TMEM lane quarter of this warp
    const int chain = blockIdx.x;         // b * nheads + h
    const int h = chain % p.nheads;
    const int b = chain / p.nheads;
    const int g = h / (p.nheads / p.ngroups);
    const int64_t L = p.seqlen;
    const uint32_t s0 = smem_u32(smem);
    float* sE = reinterpret_cast<float*>(smem + kSsdOffE);
    float* sTot = reinterpret_cast<float*>(smem + kSsdOffTot) + 4 * hp;
    const uint32_t bar0 = s0 + kSsdOffBar;
    auto bar = [bar0](int k) -> uint32_t { return bar0 + 8u * (uint32_t)k; };
    const uint32_t* tslot = reinterpret_cast<const uint32_t*>(smem + kSsdOffSlot);
    const bool has_z = p.z != nullptr;

    if (warp == 0) tmem_alloc(s0 + kSsdOffSlot, kSsdTmemCols);
    if (tid == 0) {
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_z);
        prefetch_tensormap(&tm_B);
        prefetch_tensormap(&tm_C);
        prefetch_tensormap(&tm_out);
#pragma unroll
        for (int k = 0; k < kSsdBars; ++k) mbar_init(bar(k), 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t tlane = tmem + ((uint32_t)(wq * 32) << 16);   // this warp's 32 lanes

    const float A2 = p.A[h] * kLog2e;
    const float Dh = p.D ? p.D[h] : 0.0f;
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.0f;

    // This thread holds H[q] = state[32 hp + q][r], in fp32.
    float H[kSsdP / 2];
    const size_t hoff = ((size_t)chain * kSsdP + 32 * hp) * kSsdN + r;
#pragma unroll
    for (int q = 0; q < kSsdP / 2; ++q) H[q] = p.h0 ? p.h0[hoff + (size_t)q * kSsdN] : 0.0f;
    ssd_store_state(smem, r, hp, H);
    fence_proxy_async_smem();

    const int64_t nchunks = (L + kSsdQ - 1) / kSsdQ;
    // Each mbarrier completes once per chunk, so the parity of chunk c's
    // completion is c & 1.  Threads wait (bounded) on the barriers whose data
    // they read; a CTA-wide barrier sits only where threads hand each other
    // data (4 per chunk), and it also spreads a failed wait to every thread.
    // Thread 0 issues every copy and product and tracks which completions are
    // outstanding (`pend`) and their parity (`par`, that of the chunk whose
    // data they carry): a failed CTA waits for them before it leaves.
    uint32_t pend = 0, par = 0;
    bool failed = false, lost = false;   // lost: this thread's own wait gave up
    auto issued = [&](int k, int64_t chunk) {
        pend |= 1u << k;
        par = (par & ~(1u << k)) | ((uint32_t)(chunk & 1) << k);
    };
    auto poll = [&](int k, int64_t c) {
        if (!mbar_wait_bounded(bar(k), (uint32_t)(c & 1))) lost = true;
        else if (tid == 0) pend &= ~(1u << k);
        tc_fence_after();
    };
    auto sync_failed = [&]() -> bool {   // CTA barrier; true on every thread if any wait gave up
        tc_fence_before();
        const bool f = __syncthreads_or(lost) != 0;
        tc_fence_after();
        return f;
    };
    // K-major operand, K step k of 16 columns: 32 bytes along the swizzled
    // 128-byte rows, the second 64 columns one half (16 KB) further.
    auto kmaj = [](int k) -> uint32_t { return (uint32_t)((k >> 2) * 16384 + (k & 3) * 32); };
    // dt of this row's token in the next chunk, loaded one chunk ahead (both
    // halves of a row load and compute the same values).
    auto load_dt = [&](int64_t l) -> float {
        return l < L ? __bfloat162float(p.dt[((int64_t)b * L + l) * p.nheads + h]) : 0.0f;
    };
    float dt_next = load_dt(r);

    if (nchunks > 0 && tid == 0) {
        mbar_arrive_expect_tx(bar(kBarC), 32768);
        tma_load_tile(s0 + kSsdOffC, &tm_C, 0, g, b, bar(kBarC));
        mbar_arrive_expect_tx(bar(kBarB), 32768);
        tma_load_tile(s0 + kSsdOffB, &tm_B, 0, g, b, bar(kBarB));
        mbar_arrive_expect_tx(bar(kBarX), 16384);
        tma_load_tile(s0 + kSsdOffX, &tm_x, 0, h, b, bar(kBarX));
        issued(kBarC, 0);
        issued(kBarB, 0);
        issued(kBarX, 0);
    }
    __syncthreads();   // the start state's hi/lo pair is in HX

    constexpr uint32_t id_g = umma_idesc_bf16(128, 128, false, false);
    constexpr uint32_t id_off = umma_idesc_bf16(128, 64, false, true);
    constexpr uint32_t id_s = umma_idesc_bf16(128, 64, true, true);
    constexpr uint32_t id_y = umma_idesc_bf16(128, 64, false, true);

    for (int64_t c = 0; c < nchunks; ++c) {
        const int l0 = (int)(c * kSsdQ);
        const bool more = c + 1 < nchunks;

        // ---- C landed: MMA 3, Y = C (H_hi + H_lo)^T (HX holds the entering
        // state's pair, published by the previous chunk's last barrier).
        if (tid == 0) {
            poll(kBarC, c);
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < kSsdN / 16; ++k)
                umma_bf16(tmem + kTmY, umma_sdesc_sw128(s0 + kSsdOffC + kmaj(k), 16, 1024),
                          umma_sdesc_sw128(s0 + kSsdOffHX + k * 2048, 16384, 1024), id_off, k);
#pragma unroll
            for (int k = 0; k < kSsdN / 16; ++k)
                umma_bf16(tmem + kTmY, umma_sdesc_sw128(s0 + kSsdOffC + kmaj(k), 16, 1024),
                          umma_sdesc_sw128(s0 + kSsdOffHX + kSsdLoBytes + k * 2048, 16384, 1024),
                          id_off, 1);
            umma_commit(bar(kBarYoff));
            issued(kBarYoff, c);
        }

        // ---- Delta, the running log2-decay c_i and e_i = c_i - log2(Delta_i),
        // while MMA 3 runs.
        float delta = 0.0f;
        if (l0 + r < L) {
            const float sarg = dt_next + bias;
            delta = p.softplus ? softplus_f32(sarg) : sarg;
        }
        dt_next = load_dt((int64_t)l0 + kSsdQ + r);
        float a = delta * A2;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, a, o);
            if (lane >= o) a += v;
        }
        if (lane == 31) sTot[wq] = a;
        __syncthreads();                                                 // barrier 1
        float pre = 0.0f;
        for (int w = 0; w < wq; ++w) pre += sTot[w];
        const float ci = a + pre;
        const float cQ = (sTot[0] + sTot[1]) + (sTot[2] + sTot[3]);
        const float e_own = ci - lg2_approx(delta);   // +inf for Delta = 0
        if (hp == 0) sE[r] = -e_own;                   // stored negated: c_i - e_j is an add

        // ---- x landed and MMA 3 is done with the HX buffer: Xw_j hi/lo
        // (row j = r, this half's columns), Xw_j = 2^(c_Q - e_j) x_j; and
        // Y_i = 2^(c_i) Y_i in place, onto which MMA 2 will accumulate.
        poll(kBarX, c);
        poll(kBarYoff, c);
        {
            const float w = ex2_approx(cQ - e_own);
            const float2 w2 = make_float2(w, w);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t off = ssd_sw128(r, 4 * hp + q);
                float f[8];
                unpack16(*reinterpret_cast<const uint4*>(smem + kSsdOffX + off), f);
#pragma unroll
                for (int k = 0; k < 8; k += 2) {
                    const float2 v = __fmul2_rn(make_float2(f[k], f[k + 1]), w2);
                    f[k] = v.x;
                    f[k + 1] = v.y;
                }
                uint4 hi, lo;
                split16(f, hi, lo);
                *reinterpret_cast<uint4*>(smem + kSsdOffHX + off) = hi;
                *reinterpret_cast<uint4*>(smem + kSsdOffHX + kSsdLoBytes + off) = lo;
            }
        }
        fence_proxy_async_smem();
        {
            const float sc = ex2_approx(ci);
            const float2 sc2 = make_float2(sc, sc);
            float y[32];
            tmem_ld32(tlane + kTmY + 32 * hp, y);
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
                const float2 v = __fmul2_rn(make_float2(y[k], y[k + 1]), sc2);
                y[k] = v.x;
                y[k + 1] = v.y;
            }
            tmem_st32f(tlane + kTmY + 32 * hp, y);
        }
        tmem_wait_st();

        // ---- every Xw row and e are written: MMA 4, S^T = B^T (Xw_hi + Xw_lo),
        // committed alone, then MMA 1, G = C B^T.
        if (sync_failed()) { failed = true; break; }                    // barrier 2
        if (tid == 0) {
            poll(kBarB, c);
#pragma unroll
            for (int k = 0; k < kSsdQ / 16; ++k)
                umma_bf16(tmem + kTmS, umma_sdesc_sw128(s0 + kSsdOffB + k * 2048, 16384, 1024),
                          umma_sdesc_sw128(s0 + kSsdOffHX + k * 2048, 16384, 1024), id_s, k);
#pragma unroll
            for (int k = 0; k < kSsdQ / 16; ++k)
                umma_bf16(tmem + kTmS, umma_sdesc_sw128(s0 + kSsdOffB + k * 2048, 16384, 1024),
                          umma_sdesc_sw128(s0 + kSsdOffHX + kSsdLoBytes + k * 2048, 16384, 1024),
                          id_s, 1);
            umma_commit(bar(kBarS));
#pragma unroll
            for (int k = 0; k < kSsdN / 16; ++k)
                umma_bf16(tmem + kTmG, umma_sdesc_sw128(s0 + kSsdOffC + kmaj(k), 16, 1024),
                          umma_sdesc_sw128(s0 + kSsdOffB + kmaj(k), 16, 1024), id_g, k);
            umma_commit(bar(kBarG));
            issued(kBarS, c);
            issued(kBarG, c);
        }

        // ---- state: H = 2^(c_Q) H + S (row n = r, this half's columns), in
        // registers while MMA 1 runs; its hi/lo pair goes to the HX buffer,
        // which MMA 4 no longer reads, for the next chunk's MMA 3.
        poll(kBarS, c);
        {
            const float dq = ex2_approx(cQ);
            float sv[32];
            tmem_ld32(tlane + kTmS + 32 * hp, sv);
            const float2 dq2 = make_float2(dq, dq);
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
                const float2 v = __ffma2_rn(dq2, make_float2(H[k], H[k + 1]), make_float2(sv[k], sv[k + 1]));
                H[k] = v.x;
                H[k + 1] = v.y;
            }
        }
        ssd_store_state(smem, r, hp, H);
        fence_proxy_async_smem();

        // ---- MMA 1 done: C and B are free.  Next chunk's C; this chunk's gate
        // tile into B's first half.
        poll(kBarG, c);
        if (tid == 0) {
            if (more) {
                mbar_arrive_expect_tx(bar(kBarC), 32768);
                tma_load_tile(s0 + kSsdOffC, &tm_C, l0 + kSsdQ, g, b, bar(kBarC));
                issued(kBarC, c + 1);
            }
            if (has_z) {
                mbar_arrive_expect_tx(bar(kBarZ), 16384);
                tma_load_tile(s0 + kSsdOffB, &tm_z, l0, h, b, bar(kBarZ));
                issued(kBarZ, c);
            }
        }

        // ---- Gm_ij = G_ij 2^(c_i - e_j) for j <= i (row i = r), as hi/lo pairs
        // written over the G columns they come from.  Rows [32 wq, 32 wq + 32)
        // need column quarters 0 .. wq (quarter wq straddles the diagonal); the
        // quarters above are zero.  This half takes quarters hp and hp + 2, so
        // no warp forms more than two; quarter q's lo words go to its own
        // columns 32 q .. 32 q + 15 and its hi words to 32 q + 16 .. 32 q + 31,
        // which this thread has read already and no other thread touches.
        {
            const float2 ci2 = make_float2(ci, ci);
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const int quarter = hp + 2 * s;
                uint32_t hi[16], lo[16];
                if (quarter > wq) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) hi[k] = lo[k] = 0u;
                } else {
                    float gv[32];
                    tmem_ld32(tlane + kTmG + 32 * quarter, gv);
                    const bool diag = quarter == wq;   // D_h x_i enters as Gm_ii += D_h
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int j0 = quarter * 32 + q * 8;
                        const float4 e0 = *reinterpret_cast<const float4*>(sE + j0);
                        const float4 e1 = *reinterpret_cast<const float4*>(sE + j0 + 4);
                        const float2 ne[4] = {make_float2(e0.x, e0.y), make_float2(e0.z, e0.w),
                                              make_float2(e1.x, e1.y), make_float2(e1.z, e1.w)};
                        float f[8];
#pragma unroll
                        for (int k = 0; k < 8; k += 2) {
                            const float2 arg = __fadd2_rn(ci2, ne[k / 2]);
                            const float2 v = __fmul2_rn(make_float2(gv[q * 8 + k], gv[q * 8 + k + 1]),
                                                        make_float2(ex2_approx(arg.x), ex2_approx(arg.y)));
                            f[k] = v.x;
                            f[k + 1] = v.y;
                        }
                        if (diag) {
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                f[k] = j0 + k < r ? f[k] : (j0 + k == r ? f[k] + Dh : 0.0f);
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            split_bf16x2(f[2 * k], f[2 * k + 1], hi[q * 4 + k], lo[q * 4 + k]);
                    }
                }
                tmem_st16(tlane + kTmG + 32 * quarter, lo);
                tmem_st16(tlane + kTmG + 32 * quarter + 16, hi);
            }
        }
        tmem_wait_st();

        // ---- every Gm row and the rescaled Y are in place: MMA 2,
        // Y += (Gm_hi + Gm_lo) X, A from tensor memory (K step k: columns
        // 16 k .. 16 k + 15 of quarter k / 2).
        if (sync_failed()) { failed = true; break; }                    // barrier 3
        if (tid == 0) {
#pragma unroll
            for (int k = 0; k < kSsdQ / 16; ++k)
                umma_bf16_ta(tmem + kTmY, tmem + kTmG + 32 * (k >> 1) + 16 + 8 * (k & 1),
                             umma_sdesc_sw128(s0 + kSsdOffX + k * 2048, 16384, 1024), id_y, 1);
#pragma unroll
            for (int k = 0; k < kSsdQ / 16; ++k)
                umma_bf16_ta(tmem + kTmY, tmem + kTmG + 32 * (k >> 1) + 8 * (k & 1),
                             umma_sdesc_sw128(s0 + kSsdOffX + k * 2048, 16384, 1024), id_y, 1);
            umma_commit(bar(kBarYd));
            issued(kBarYd, c);
        }
        poll(kBarYd, c);
        if (has_z) poll(kBarZ, c);

        // ---- y_i = Y_i (row i = r, this half's columns), gated, written as
        // bf16 over the x tile (no longer read), then stored by TMA (rows past
        // the end dropped).
        {
            float y[32];
            tmem_ld32(tlane + kTmY + 32 * hp, y);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t off = ssd_sw128(r, 4 * hp + q);
                float f[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) f[k] = y[q * 8 + k];
                if (has_z) {
                    // silu(z) = z / (1 + 2^(-z log2 e)), two lanes at a time
                    float zv[8];
                    unpack16(*reinterpret_cast<const uint4*>(smem + kSsdOffB + off), zv);
#pragma unroll
                    for (int k = 0; k < 8; k += 2) {
                        const float2 z2 = make_float2(zv[k], zv[k + 1]);
                        const float2 t = __fmul2_rn(z2, make_float2(-kLog2e, -kLog2e));
                        const float2 d = __fadd2_rn(make_float2(ex2_approx(t.x), ex2_approx(t.y)),
                                                    make_float2(1.0f, 1.0f));
                        const float2 g2 = __fmul2_rn(z2, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
                        const float2 v = __fmul2_rn(make_float2(f[k], f[k + 1]), g2);
                        f[k] = v.x;
                        f[k + 1] = v.y;
                    }
                }
                *reinterpret_cast<uint4*>(smem + kSsdOffX + off) = pack16(f);
            }
        }
        fence_proxy_async_smem();
        if (sync_failed()) { failed = true; break; }                    // barrier 4
        // The gate tile is consumed: thread 0 requests the next chunk's B and
        // moves on.  Thread kSsdStoreThread stores the output tile and, once
        // the store has read it, requests the next chunk's x into it.
        if (tid == 0 && more) {
            mbar_arrive_expect_tx(bar(kBarB), 32768);
            tma_load_tile(s0 + kSsdOffB, &tm_B, l0 + kSsdQ, g, b, bar(kBarB));
            issued(kBarB, c + 1);
        }
        if (tid == kSsdStoreThread) {
            tma_store_tile(&tm_out, s0 + kSsdOffX, l0, h, b);
            bulk_commit();
            if (more) {
                bulk_wait_read<0>();
                mbar_arrive_expect_tx(bar(kBarX), 16384);
                tma_load_tile(s0 + kSsdOffX, &tm_x, l0 + kSsdQ, h, b, bar(kBarX));
            }
        }
        if (tid == 0 && more) issued(kBarX, c + 1);
    }

    if (!failed && p.hT) {
#pragma unroll
        for (int q = 0; q < kSsdP / 2; ++q) p.hT[hoff + (size_t)q * kSsdN] = H[q];
    }
    if (tid == kSsdStoreThread) bulk_wait<0>();   // output stores done before shared memory goes
    if (tid == 0) {
        // After a timeout, wait (bounded) for every copy and product still in
        // flight, so that none lands in shared or tensor memory after the CTA
        // has released them.
        if (failed) {
#pragma unroll 1
            for (int k = 0; k < kSsdBars; ++k)
                if ((pend >> k) & 1u) (void)mbar_wait_bounded(bar(k), (par >> k) & 1u);
        }
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
