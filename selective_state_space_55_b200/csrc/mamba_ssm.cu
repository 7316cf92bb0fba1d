// C ABI of the selective-SSM library: argument validation, planning, TMA
// descriptor set-up and kernel dispatch.  One translation unit holds every
// kernel so that device globals need no separate device link.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "mamba_ssm.h"
#include "selective_scan.cuh"
#include "state_update.cuh"
#include "conv1d.cuh"
#include "scan_backward.cuh"
#include "ssd_chunk_scan.cuh"
#include "scan_carry.cuh"
#include "scan_split.cuh"

namespace mamba {

namespace {

constexpr int kMaxDevices = 64;

int dtype_bytes(int32_t dt) { return dt == MAMBA_BF16 ? 2 : 4; }
bool dtype_ok(int32_t dt) { return dt == MAMBA_F32 || dt == MAMBA_BF16; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

mamba_status_t check_dims(const mamba_dims_t* dims, bool scan) {
    if (dims == nullptr) return MAMBA_ERR_INVALID_ARG;
    if (dims->batch < 0 || dims->dim < 0 || dims->dstate < 0) return MAMBA_ERR_INVALID_ARG;
    if (scan && dims->seqlen < 0) return MAMBA_ERR_INVALID_ARG;
    if (scan && dims->num_chunks < 0) return MAMBA_ERR_INVALID_ARG;
    if (dims->dstate < 1 || dims->dstate > MAMBA_MAX_DSTATE) return MAMBA_ERR_UNSUPPORTED;
    if (!dtype_ok(dims->io_dtype) || !dtype_ok(dims->bc_dtype)) return MAMBA_ERR_UNSUPPORTED;
    // Index arithmetic inside the kernels is 64-bit; TMA coordinates are
    // 32-bit, so keep every extent below 2^31.
    const int64_t lim = (int64_t)1 << 31;
    if (dims->batch >= lim || dims->dim >= lim || (scan && dims->seqlen >= lim))
        return MAMBA_ERR_INVALID_ARG;
    return MAMBA_OK;
}

// SM count of the current device, cached per device.
int current_sm_count(int* device_out) {
    static int cached[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (device_out) *device_out = dev;
    if (dev >= 0 && dev < kMaxDevices && cached[dev] > 0) return cached[dev];
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    if (dev >= 0 && dev < kMaxDevices) cached[dev] = sms;
    return sms;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 3-D map over a row-major (d2, d1, d0) tensor, d0 innermost, box (box0, box1, 1).
bool encode_map_3d(CUtensorMap* map, const void* base, int esize, uint64_t d0, uint64_t d1,
                   uint64_t d2, uint32_t box0, uint32_t box1, CUtensorMapSwizzle swizzle) {
    auto encode = tensor_map_encoder();
    if (encode == nullptr) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * esize, d0 * d1 * esize};
    const cuuint32_t box[3] = {box0, box1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt =
        esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const CUresult r = encode(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <typename Kernel>
cudaError_t ensure_smem_attr(Kernel kernel, int bytes, bool* done_per_device, int dev) {
    if (dev >= 0 && dev < kMaxDevices && done_per_device[dev]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done_per_device[dev] = true;
    return e;
}

template <typename IoT, int kCpl, bool kHasZ, bool kSoftplus, bool kZoh, bool kBld, bool kLookback>
cudaError_t launch_scan(const ScanParams& prm, const CUtensorMap* maps, int64_t want_warps,
                        int dev, int sms, cudaStream_t stream) {
    using Lay = ScanLayout<kCpl>;
    static bool attr_done[kMaxDevices] = {false};
    static int resident[kMaxDevices] = {0};
    auto kernel = selective_scan_fwd_kernel<IoT, kCpl, kHasZ, kSoftplus, kZoh, kBld, kLookback>;
    cudaError_t e = ensure_smem_attr(kernel, Lay::kCtaSmem, attr_done, dev);
    if (e != cudaSuccess) return e;
    int per_sm = (dev >= 0 && dev < kMaxDevices) ? resident[dev] : 0;
    if (per_sm <= 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kScanWarps * 32,
                                                          Lay::kCtaSmem);
        if (e != cudaSuccess) return e;
        if (per_sm <= 0) return cudaErrorInvalidConfiguration;
        if (dev >= 0 && dev < kMaxDevices) resident[dev] = per_sm;
    }
    // Persistent grid: every warp keeps pulling work items until none are left.
    const int64_t want = (want_warps + kScanWarps - 1) / kScanWarps;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)per_sm * sms));
    kernel<<<(unsigned)grid, kScanWarps * 32, Lay::kCtaSmem, stream>>>(prm, maps[0], maps[1],
                                                                         maps[2], maps[3], maps[4]);
    return cudaGetLastError();
}

template <typename IoT, int kCpl, bool kZoh, bool kBld, bool kLookback>
cudaError_t dispatch_scan_cpl(const ScanParams& prm, const CUtensorMap* maps, bool has_z, bool sp,
                              int64_t want_warps, int dev, int sms, cudaStream_t stream) {
    if (has_z)
        return sp ? launch_scan<IoT, kCpl, true, true, kZoh, kBld, kLookback>(prm, maps, want_warps, dev, sms, stream)
                  : launch_scan<IoT, kCpl, true, false, kZoh, kBld, kLookback>(prm, maps, want_warps, dev, sms, stream);
    return sp ? launch_scan<IoT, kCpl, false, true, kZoh, kBld, kLookback>(prm, maps, want_warps, dev, sms, stream)
              : launch_scan<IoT, kCpl, false, false, kZoh, kBld, kLookback>(prm, maps, want_warps, dev, sms, stream);
}

template <typename IoT, bool kHasZ, bool kSoftplus>
cudaError_t launch_scan_split(const ScanParams& prm, const CUtensorMap* maps, int64_t want_warps,
                              int dev, int sms, cudaStream_t stream) {
    using Lay = SplitLayout;
    static bool attr_done[kMaxDevices] = {false};
    static int resident[kMaxDevices] = {0};
    auto kernel = selective_scan_fwd_split_kernel<IoT, kHasZ, kSoftplus>;
    cudaError_t e = ensure_smem_attr(kernel, Lay::kCtaSmem, attr_done, dev);
    if (e != cudaSuccess) return e;
    int per_sm = (dev >= 0 && dev < kMaxDevices) ? resident[dev] : 0;
    if (per_sm <= 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, Lay::kWarps * 32,
                                                          Lay::kCtaSmem);
        if (e != cudaSuccess) return e;
        if (per_sm <= 0) return cudaErrorInvalidConfiguration;
        if (dev >= 0 && dev < kMaxDevices) resident[dev] = per_sm;
    }
    const int64_t want = (want_warps + Lay::kWarps - 1) / Lay::kWarps;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)per_sm * sms));
    kernel<<<(unsigned)grid, Lay::kWarps * 32, Lay::kCtaSmem, stream>>>(prm, maps[0], maps[1],
                                                                          maps[2], maps[3], maps[4]);
    return cudaGetLastError();
}

// Two lanes per channel (chained mode, Euler, (batch, dim, seqlen)).
template <typename IoT>
cudaError_t dispatch_scan_split(const ScanParams& prm, const CUtensorMap* maps, bool has_z, bool sp,
                                int64_t want_warps, int dev, int sms, cudaStream_t stream) {
    if (has_z)
        return sp ? launch_scan_split<IoT, true, true>(prm, maps, want_warps, dev, sms, stream)
                  : launch_scan_split<IoT, true, false>(prm, maps, want_warps, dev, sms, stream);
    return sp ? launch_scan_split<IoT, false, true>(prm, maps, want_warps, dev, sms, stream)
              : launch_scan_split<IoT, false, false>(prm, maps, want_warps, dev, sms, stream);
}

// Kernel instance for (channels per lane, zero-order hold, activation layout, look-back).
template <typename IoT>
cudaError_t dispatch_scan(const ScanParams& prm, const CUtensorMap* maps, int cpl, bool has_z,
                          bool sp, bool zoh, int64_t want_warps, int dev, int sms,
                          cudaStream_t stream) {
    if (cpl != 1) return cudaErrorInvalidValue;
    if (prm.bld)
        return zoh ? dispatch_scan_cpl<IoT, 1, true, true, false>(prm, maps, has_z, sp, want_warps, dev, sms, stream)
                   : dispatch_scan_cpl<IoT, 1, false, true, false>(prm, maps, has_z, sp, want_warps, dev, sms, stream);
    if (prm.mode == kModeLookback)
        return zoh ? dispatch_scan_cpl<IoT, 1, true, false, true>(prm, maps, has_z, sp, want_warps, dev, sms, stream)
                   : dispatch_scan_cpl<IoT, 1, false, false, true>(prm, maps, has_z, sp, want_warps, dev, sms, stream);
    return zoh ? dispatch_scan_cpl<IoT, 1, true, false, false>(prm, maps, has_z, sp, want_warps, dev, sms, stream)
               : dispatch_scan_cpl<IoT, 1, false, false, false>(prm, maps, has_z, sp, want_warps, dev, sms, stream);
}

// Correction pass of the parallel mode: a persistent grid of warps that pull
// (chain, segment) items from a counter; items are few and uneven in length
// (each stops where its start state has decayed below fp32's range).
template <typename IoT, typename BcT, bool kHasZ, bool kSoftplus>
cudaError_t launch_correct(const CorrectParams& q, int dev, int sms, cudaStream_t stream) {
    static int resident[kMaxDevices] = {0};
    auto kernel = scan_correct_kernel<IoT, BcT, kHasZ, kSoftplus>;
    int per_sm = (dev >= 0 && dev < kMaxDevices) ? resident[dev] : 0;
    if (per_sm <= 0) {
        const cudaError_t e =
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kCorrectWarps * 32, 0);
        if (e != cudaSuccess) return e;
        if (per_sm <= 0) return cudaErrorInvalidConfiguration;
        if (dev >= 0 && dev < kMaxDevices) resident[dev] = per_sm;
    }
    const int64_t need = (q.items + kCorrectWarps - 1) / kCorrectWarps;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((int64_t)per_sm * sms, need));
    kernel<<<(unsigned)grid, kCorrectWarps * 32, 0, stream>>>(q);
    return cudaGetLastError();
}

template <typename IoT>
cudaError_t dispatch_correct(const CorrectParams& q, bool has_z, bool sp, int dev, int sms,
                             cudaStream_t stream) {
    if (q.bc_bf16) {
        if (has_z)
            return sp ? launch_correct<IoT, __nv_bfloat16, true, true>(q, dev, sms, stream)
                      : launch_correct<IoT, __nv_bfloat16, true, false>(q, dev, sms, stream);
        return sp ? launch_correct<IoT, __nv_bfloat16, false, true>(q, dev, sms, stream)
                  : launch_correct<IoT, __nv_bfloat16, false, false>(q, dev, sms, stream);
    }
    if (has_z)
        return sp ? launch_correct<IoT, float, true, true>(q, dev, sms, stream)
                  : launch_correct<IoT, float, true, false>(q, dev, sms, stream);
    return sp ? launch_correct<IoT, float, false, true>(q, dev, sms, stream)
              : launch_correct<IoT, float, false, false>(q, dev, sms, stream);
}

template <typename IoT, typename BcT, bool kHasZ, bool kZoh>
cudaError_t launch_update_bulk(const UpdateParams& prm, int dev, int sms, bool pdl,
                               cudaStream_t stream) {
    static bool attr_done[kMaxDevices] = {false};
    static int resident[kMaxDevices] = {0};
    auto kernel = pdl ? state_update_bulk_kernel<IoT, BcT, kHasZ, kZoh, true>
                      : state_update_bulk_kernel<IoT, BcT, kHasZ, kZoh, false>;
    static bool attr_done_pdl[kMaxDevices] = {false};
    static int resident_pdl[kMaxDevices] = {0};
    bool* done = pdl ? attr_done_pdl : attr_done;
    int* res = pdl ? resident_pdl : resident;
    cudaError_t e = ensure_smem_attr(kernel, kBulkSmemBytes, done, dev);
    if (e != cudaSuccess) return e;
    int per_sm = (dev >= 0 && dev < kMaxDevices) ? res[dev] : 0;
    if (per_sm <= 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kBulkThreads,
                                                          kBulkSmemBytes);
        if (e != cudaSuccess) return e;
        if (per_sm <= 0) return cudaErrorInvalidConfiguration;
        if (dev >= 0 && dev < kMaxDevices) res[dev] = per_sm;
    }
    // Each CTA owns one channel block and every J-th batch row: J copies of the
    // nblk blocks fill the resident CTAs.  Among J <= resident / nblk pick the
    // one whose slowest CTA has the fewest rows, then the smallest such J.
    const int64_t nblk = (prm.dim + kBulkTile - 1) / kBulkTile;
    const int64_t jmax = std::max<int64_t>(1, std::min<int64_t>(prm.batch, ((int64_t)per_sm * sms) / nblk));
    int64_t J = jmax;
    for (int64_t j = jmax; j >= 1 && j * 2 >= jmax; --j)
        if ((prm.batch + j - 1) / j <= (prm.batch + J - 1) / J) J = j;
    const int64_t grid = nblk * J;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kBulkThreads);
    cfg.dynamicSmemBytes = kBulkSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kernel, prm);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename IoT, typename BcT>
cudaError_t dispatch_update_bc(const UpdateParams& prm, bool fast, bool bulk, bool has_z,
                               int dev, int sms, bool pdl, cudaStream_t stream) {
    if (bulk) {
        if (prm.zoh)
            return has_z ? launch_update_bulk<IoT, BcT, true, true>(prm, dev, sms, pdl, stream)
                         : launch_update_bulk<IoT, BcT, false, true>(prm, dev, sms, pdl, stream);
        return has_z ? launch_update_bulk<IoT, BcT, true, false>(prm, dev, sms, pdl, stream)
                     : launch_update_bulk<IoT, BcT, false, false>(prm, dev, sms, pdl, stream);
    }
    if (fast) {
        // x covers channels (kUpdateChainsPerCta per CTA), y covers batch rows.
        const dim3 grid((unsigned)((prm.dim + kUpdateChainsPerCta - 1) / kUpdateChainsPerCta),
                        (unsigned)std::min<int64_t>(prm.batch, 65535));
        if (has_z)
            state_update_n16_kernel<IoT, BcT, true><<<grid, kUpdateThreads, 0, stream>>>(prm);
        else
            state_update_n16_kernel<IoT, BcT, false><<<grid, kUpdateThreads, 0, stream>>>(prm);
    } else {
        const unsigned grid = (unsigned)((prm.chains + kUpdateThreads - 1) / kUpdateThreads);
        if (has_z)
            state_update_generic_kernel<IoT, BcT, true><<<grid, kUpdateThreads, 0, stream>>>(prm);
        else
            state_update_generic_kernel<IoT, BcT, false><<<grid, kUpdateThreads, 0, stream>>>(prm);
    }
    return cudaGetLastError();
}

template <typename IoT>
cudaError_t dispatch_update(const UpdateParams& prm, bool bc_bf16, bool fast, bool bulk,
                            bool has_z, int dev, int sms, bool pdl, cudaStream_t stream) {
    return bc_bf16
               ? dispatch_update_bc<IoT, __nv_bfloat16>(prm, fast, bulk, has_z, dev, sms, pdl, stream)
               : dispatch_update_bc<IoT, float>(prm, fast, bulk, has_z, dev, sms, pdl, stream);
}

}  // namespace

// Scratch layout of one scan call (offsets in bytes).
struct ScanWorkspace {
    size_t zeroed;      // prefix cleared before every call: counters and flags
    size_t carry;       // chained mode: [chains][16] fp32
    size_t ws_h;        // parallel mode: [K][chains][16] fp32
    size_t ws_sdt;      // parallel mode: [K][chains] fp32
    size_t total;
};

ScanWorkspace scan_workspace_layout(const mamba_dims_t* dims, int64_t groups, int64_t K, int mode) {
    ScanWorkspace w{};
    const size_t chains = (size_t)dims->batch * (size_t)dims->dim;
    const size_t nflags = (size_t)groups * (mode == 2 ? (size_t)K : 1);   // mode 2: one per segment
    w.zeroed = kWsFlags + align256(nflags * sizeof(unsigned int));
    size_t off = w.zeroed;
    if (mode == 0 && K > 1) {
        w.carry = off;
        off += align256(chains * kNPad * sizeof(float));
    }
    if (mode >= 1) {
        w.ws_h = off;
        off += align256((size_t)K * chains * kNPad * sizeof(float));
        w.ws_sdt = off;
        off += align256((size_t)K * chains * sizeof(float));
    }
    w.total = off;
    return w;
}

// Planning rules (pure host logic, see mamba_selective_scan_plan).
//  - One channel per lane (32-channel groups), or two (see the last rule).
//  - W = resident warps on the GPU (16 per SM), G = channel groups.
//  - G >= W/4: chained mode, K segments so that G*K is about 8 W work items
//    (even load across SMs), segments at least 256 steps long.  At most G
//    warps run, so a warp rarely picks up a segment whose predecessor has not
//    finished.
//  - G < W/4: parallel mode, K = W/G segments (one segment per resident
//    warp, so the first launch ends in one wave), segments at least 16 tiles
//    and 512 steps long.
//  - num_chunks >= 1 forces K; MAMBA_FLAG_PARALLEL_CHUNKS forces the parallel
//    mode for a forced K.
//  - Activations in the (batch, seqlen, dim) layout always run chained (the
//    correction pass reads rows along time).
//  - Chained with G < W (groups of 32 that leave resident warps idle), Euler,
//    (batch, dim, seqlen): two lanes per channel, groups of 16 (2 G warps);
//    K is then chosen for those groups.  MAMBA_FLAG_ONE_LANE_PER_CHANNEL
//    keeps one lane.
mamba_status_t plan_scan(const mamba_dims_t* dims, int sm_count, mamba_scan_plan_t* plan) {
    mamba_status_t st = check_dims(dims, true);
    if (st != MAMBA_OK) return st;
    if (plan == nullptr || sm_count <= 0) return MAMBA_ERR_INVALID_ARG;
    const bool bld = (dims->flags & MAMBA_FLAG_LAYOUT_BLD) != 0;
    if (bld && dims->num_chunks >= 1 && (dims->flags & MAMBA_FLAG_PARALLEL_CHUNKS))
        return MAMBA_ERR_UNSUPPORTED;
    *plan = mamba_scan_plan_t{};
    const int io_es = dtype_bytes(dims->io_dtype);
    const int bc_es = dtype_bytes(dims->bc_dtype);
    const int64_t T = kRowBytes / io_es;
    const int64_t L = dims->seqlen;
    const int64_t g1 = dims->batch * ((dims->dim + 31) / 32);
    const int64_t g2 = dims->batch * ((dims->dim + 63) / 64);
    const int64_t w1 = (int64_t)sm_count * ScanLayout<1>::kWarpsPerSm;
    const int64_t w2 = (int64_t)sm_count * ScanLayout<2>::kWarpsPerSm;
    // One channel per lane: measured faster than two on every workload shape
    // (16 resident warps per SM against 12; the packed fp32x2 step already
    // leaves issue slots to spare).
    const int cpl = 1;
    (void)g2;
    (void)w2;
    const int64_t groups = g1;
    const int64_t W = w1;
    plan->tile_len = (int32_t)T;
    plan->groups = groups;
    plan->warps_per_cta = kScanWarps;
    plan->channels_per_lane = cpl;
    const int64_t act_row = bld ? dims->dim : L;   // elements of an activation row
    plan->tma_capable = (L > 0 && (act_row * io_es) % 16 == 0 && (L * bc_es) % 16 == 0) ? 1 : 0;

    int64_t K = 1;
    int mode = 0;
    if (dims->num_chunks >= 1) {
        K = dims->num_chunks;
        mode = (dims->flags & MAMBA_FLAG_PARALLEL_CHUNKS) ? 1 : 0;
    } else if (groups > 0 && L > 0) {
        if (4 * groups >= W || bld) {
            const int64_t want = (8 * W + groups - 1) / groups;
            K = std::max<int64_t>(1, std::min<int64_t>(want, L / 256));
        } else {
            mode = 1;
            K = std::max<int64_t>(
                1, std::min<int64_t>(W / groups, L / std::max<int64_t>(16 * T, 512)));
        }
    }
    auto segments = [&](int64_t& k, int64_t& len) {
        len = L;
        if (k > 1 && L > 0) {
            len = ((L + k - 1) / k + T - 1) / T * T;
            k = (L + len - 1) / len;
        }
        if (k <= 1) {
            k = 1;
            len = L;
        }
    };
    int64_t seg_len = L;
    segments(K, seg_len);
    if (K == 1) mode = 0;
    if (mode == 1 && (dims->flags & MAMBA_FLAG_PARALLEL_ONE_LAUNCH)) mode = 2;
    // Two lanes per channel: chained, groups of 32 fewer than resident warps.
    int lanes = 1;
    int64_t groups_run = groups;
    if (mode == 0 && groups > 0 && L > 0 && groups < W && !bld &&
        !(dims->flags & MAMBA_FLAG_ZOH) && !(dims->flags & MAMBA_FLAG_ONE_LANE_PER_CHANNEL)) {
        lanes = 2;
        groups_run = dims->batch * ((dims->dim + 15) / 16);
        if (dims->num_chunks < 1) {
            // About 4 segments per resident warp of the two-lane kernel (8 x 4096
            // x 2048: K = 4, measured faster than 8 or 12; 6 leaves a short
            // last segment).
            const int64_t W2 = (int64_t)sm_count * SplitLayout::kWarpsPerSm;
            K = std::max<int64_t>(1, std::min<int64_t>((4 * W2 + groups_run - 1) / groups_run,
                                                       L / 256));
            segments(K, seg_len);
        }
    }
    const int64_t items = groups_run * K;
    const int64_t chains = dims->batch * dims->dim;
    const int64_t fixes = mode == 0 ? 0 : chains * (K - 1);
    if (items >= ((int64_t)1 << 31) || fixes >= ((int64_t)1 << 31)) return MAMBA_ERR_UNSUPPORTED;
    plan->groups = groups_run;
    plan->lanes_per_channel = lanes;
    plan->nchunks = (int32_t)K;
    plan->chunk_len = seg_len;
    plan->mode = mode;
    plan->units_pass_a = items;
    plan->units_pass_b = fixes;
    // Warps the persistent grid holds at once (the two-lane kernel runs
    // fewer per SM: SplitLayout::kWarpsPerSm).
    const int64_t W_run = lanes == 2 ? (int64_t)sm_count * SplitLayout::kWarpsPerSm : W;
    plan->max_warps = mode == 0 && K > 1 ? std::min<int64_t>(groups_run, W_run)
                                         : std::min<int64_t>(items, W_run);
    plan->launches = (groups > 0 && L > 0) ? (mode == 1 ? 3 : 1) : 0;
    plan->workspace_bytes =
        (groups > 0 && L > 0) ? scan_workspace_layout(dims, groups_run, K, mode).total : 0;
    return MAMBA_OK;
}

}  // namespace mamba

using namespace mamba;

mamba_status_t scan_fwd_internal(const void* u, const void* delta, const float* A, const void* B,
                                 const void* C, const float* D, const void* z,
                                 const float* delta_bias, int softplus,
                                 const float* initial_state, void* out, float* last_state,
                                 const mamba_dims_t* dims, cudaStream_t stream, float* ckpt,
                                 int64_t ckpt_tiles);

extern "C" {

MAMBA_API mamba_status_t mamba_selective_scan_plan(const mamba_dims_t* dims, int sm_count,
                                                   mamba_scan_plan_t* plan) {
    return plan_scan(dims, sm_count, plan);
}

MAMBA_API size_t mamba_selective_scan_workspace_bytes(const mamba_dims_t* dims) {
    const int sms = current_sm_count(nullptr);
    if (sms <= 0) return static_cast<size_t>(-1);
    mamba_scan_plan_t plan;
    if (plan_scan(dims, sms, &plan) != MAMBA_OK) return static_cast<size_t>(-1);
    return plan.workspace_bytes;
}

MAMBA_API mamba_status_t mamba_selective_scan_fwd(const void* u, const void* delta, const float* A,
                                                  const void* B, const void* C, const float* D,
                                                  const void* z, const float* delta_bias,
                                                  int softplus, void* out, float* last_state,
                                                  const mamba_dims_t* dims, cudaStream_t stream) {
    return mamba_selective_scan_fwd_with_state(u, delta, A, B, C, D, z, delta_bias, softplus,
                                               nullptr, out, last_state, dims, stream);
}

MAMBA_API mamba_status_t mamba_selective_scan_fwd_with_state(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus,
    const float* initial_state, void* out, float* last_state, const mamba_dims_t* dims,
    cudaStream_t stream) {
    return scan_fwd_internal(u, delta, A, B, C, D, z, delta_bias, softplus, initial_state, out,
                             last_state, dims, stream, nullptr, 0);
}

}  // extern "C"

// The forward scan.  With `ckpt` set it is the backward's checkpoint pass: no
// output, the state before every kCkptSteps steps stored to
// ckpt[chain][ckpt_tiles][16] instead.
mamba_status_t scan_fwd_internal(const void* u, const void* delta, const float* A, const void* B,
                                 const void* C, const float* D, const void* z,
                                 const float* delta_bias, int softplus,
                                 const float* initial_state, void* out, float* last_state,
                                 const mamba_dims_t* dims, cudaStream_t stream, float* ckpt,
                                 int64_t ckpt_tiles) {
    mamba_status_t st = check_dims(dims, true);
    if (st != MAMBA_OK) return st;
    const bool bld = (dims->flags & MAMBA_FLAG_LAYOUT_BLD) != 0;
    // Empty problems first: tensors without elements may have null pointers.
    const int64_t chains = dims->batch * dims->dim;
    if (chains == 0) return MAMBA_OK;
    const size_t state_bytes = (size_t)chains * dims->dstate * sizeof(float);
    if (initial_state != nullptr && !aligned(initial_state, 4)) return MAMBA_ERR_ALIGN;
    // The start state may be the last_state buffer itself (in-place
    // continuation), but must not partly overlap it.
    if (initial_state != nullptr && last_state != nullptr && initial_state != last_state) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(initial_state);
        const uintptr_t b = reinterpret_cast<uintptr_t>(last_state);
        if (a < b + state_bytes && b < a + state_bytes) return MAMBA_ERR_INVALID_ARG;
    }
    if (dims->seqlen == 0) {
        if (last_state == nullptr) return MAMBA_OK;
        if (!aligned(last_state, 4)) return MAMBA_ERR_ALIGN;
        cudaError_t e = cudaSuccess;
        if (initial_state == nullptr)
            e = cudaMemsetAsync(last_state, 0, state_bytes, stream);
        else if (initial_state != last_state)
            e = cudaMemcpyAsync(last_state, initial_state, state_bytes, cudaMemcpyDeviceToDevice,
                                stream);
        return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
    }
    if (u == nullptr || delta == nullptr || A == nullptr || B == nullptr || C == nullptr ||
        (out == nullptr && ckpt == nullptr))
        return MAMBA_ERR_INVALID_ARG;
    const int io_es = dtype_bytes(dims->io_dtype);
    const int bc_es = dtype_bytes(dims->bc_dtype);
    if (!aligned(u, io_es) || !aligned(delta, io_es) || (out && !aligned(out, io_es)) ||
        (z && !aligned(z, io_es)) || !aligned(B, bc_es) || !aligned(C, bc_es) || !aligned(A, 4) ||
        (D && !aligned(D, 4)) || (delta_bias && !aligned(delta_bias, 4)) ||
        (last_state && !aligned(last_state, 4)))
        return MAMBA_ERR_ALIGN;

    int dev = 0;
    const int sms = current_sm_count(&dev);
    if (sms <= 0) return MAMBA_ERR_CUDA;
    mamba_scan_plan_t plan;
    mamba_dims_t pd = *dims;
    if (ckpt != nullptr) pd.flags |= MAMBA_FLAG_ONE_LANE_PER_CHANNEL;   // checkpoints: one lane
    st = plan_scan(&pd, sms, &plan);
    if (st != MAMBA_OK) return st;
    if (dims->workspace == nullptr || dims->workspace_bytes < plan.workspace_bytes)
        return MAMBA_ERR_WORKSPACE;
    const int64_t group_rows = 32 / plan.lanes_per_channel;
    if (!aligned(dims->workspace, 256)) return MAMBA_ERR_ALIGN;

    ScanParams prm{};
    prm.u = u;
    prm.delta = delta;
    prm.z = z;
    prm.A = A;
    prm.B = B;
    prm.C = C;
    prm.D = D;
    prm.delta_bias = delta_bias;
    prm.out = out;
    prm.last_state = last_state;
    prm.h0 = initial_state;
    prm.ckpt = ckpt;
    prm.ckpt_tiles = ckpt_tiles;
    prm.batch = dims->batch;
    prm.dim = dims->dim;
    prm.seqlen = dims->seqlen;
    prm.groups_per_batch = (dims->dim + group_rows - 1) / group_rows;
    prm.groups = plan.groups;
    prm.chains = chains;
    prm.seg_len = plan.chunk_len;
    prm.dstate = (int)dims->dstate;
    prm.nseg = plan.nchunks;
    prm.bc_bf16 = dims->bc_dtype == MAMBA_BF16;
    prm.bld = bld ? 1 : 0;
    prm.out_step = bld ? dims->dim : 1;
    prm.vec_out = !bld && out != nullptr && ((dims->seqlen * io_es) % 16 == 0) && aligned(out, 16);
    prm.vec_io = ((dims->seqlen * io_es) % 16 == 0) && aligned(delta, 16) && out != nullptr &&
                 aligned(out, 16) && (!z || aligned(z, 16));
    prm.vec_c = ((dims->seqlen * bc_es) % 16 == 0) && aligned(C, 16);
    // A predecessor segment legitimately takes well under 64 us per step even
    // on a crowded GPU; wait that long (at least ~1 s) before reporting a stall.
    prm.withhold_handoff = (dims->flags & MAMBA_FLAG_TEST_WITHHOLD_HANDOFF) ? 1 : 0;
    prm.flag_poll_limit =
        prm.withhold_handoff
            ? (1u << 18)
            : (unsigned int)std::min<int64_t>(std::max<int64_t>(plan.chunk_len * 64, 1 << 20),
                                              (int64_t)1 << 31);
    uint8_t* ws = static_cast<uint8_t*>(dims->workspace);
    const ScanWorkspace lay = scan_workspace_layout(&pd, plan.groups, plan.nchunks, plan.mode);
    unsigned int* counters = reinterpret_cast<unsigned int*>(ws + kWsCounters);
    prm.flags = reinterpret_cast<unsigned int*>(ws + kWsFlags);
    if (lay.carry) prm.carry = reinterpret_cast<float*>(ws + lay.carry);
    if (lay.ws_h) prm.ws_h = reinterpret_cast<float*>(ws + lay.ws_h);
    if (lay.ws_sdt) prm.ws_sdt = reinterpret_cast<float*>(ws + lay.ws_sdt);

    const bool use_tma = plan.tma_capable && !(dims->flags & MAMBA_FLAG_NO_TMA) &&
                         aligned(u, 16) && aligned(delta, 16) && (!z || aligned(z, 16)) &&
                         aligned(B, 16) && aligned(C, 16) && tensor_map_encoder() != nullptr;
    prm.use_tma = use_tma ? 1 : 0;
    CUtensorMap maps[5];
    std::memset(maps, 0, sizeof(maps));
    if (use_tma) {
        const uint32_t T = (uint32_t)plan.tile_len;
        const uint64_t L = (uint64_t)dims->seqlen;
        const uint64_t Dm = (uint64_t)dims->dim, Bt = (uint64_t)dims->batch;
        const uint64_t N = (uint64_t)dims->dstate;
        const uint32_t rows = (uint32_t)group_rows;
        // (rows x T) tiles of (batch, dim, seqlen) rows with 32-byte swizzle, or
        // dense (T x rows) tiles of (batch, seqlen, dim) that the kernel transposes
        auto act = [&](CUtensorMap* m, const void* base) {
            return bld ? encode_map_3d(m, base, io_es, Dm, L, Bt, rows, T, CU_TENSOR_MAP_SWIZZLE_NONE)
                       : encode_map_3d(m, base, io_es, L, Dm, Bt, T, rows, CU_TENSOR_MAP_SWIZZLE_32B);
        };
        bool ok = act(&maps[0], u) && act(&maps[1], delta) && act(&maps[2], z ? z : u) &&
                  encode_map_3d(&maps[3], B, bc_es, L, N, Bt, T, (uint32_t)N,
                                CU_TENSOR_MAP_SWIZZLE_NONE) &&
                  encode_map_3d(&maps[4], C, bc_es, L, N, Bt, T, (uint32_t)N,
                                CU_TENSOR_MAP_SWIZZLE_NONE);
        if (!ok) {
            prm.use_tma = 0;
            std::memset(maps, 0, sizeof(maps));
        }
    }

    // Counters and flags start at zero on every call.
    if (cudaMemsetAsync(ws, 0, lay.zeroed, stream) != cudaSuccess) return MAMBA_ERR_CUDA;
    const bool has_z = z != nullptr;
    const bool sp = softplus != 0;
    const bool zoh = (dims->flags & MAMBA_FLAG_ZOH) != 0;
    auto run = [&](int mode, unsigned int* counter, int64_t items) -> cudaError_t {
        prm.mode = mode;
        prm.counter = counter;
        prm.items = items;
        if (items == 0) return cudaSuccess;
        if (plan.lanes_per_channel == 2)
            return dims->io_dtype == MAMBA_BF16
                       ? dispatch_scan_split<__nv_bfloat16>(prm, maps, has_z, sp, plan.max_warps,
                                                            dev, sms, stream)
                       : dispatch_scan_split<float>(prm, maps, has_z, sp, plan.max_warps, dev,
                                                    sms, stream);
        return dims->io_dtype == MAMBA_BF16
                   ? dispatch_scan<__nv_bfloat16>(prm, maps, plan.channels_per_lane, has_z, sp,
                                                  zoh, plan.max_warps, dev, sms, stream)
                   : dispatch_scan<float>(prm, maps, plan.channels_per_lane, has_z, sp, zoh,
                                          plan.max_warps, dev, sms, stream);
    };
    cudaError_t e;
    if (plan.mode == 0) {
        e = run(kModeChained, counters, plan.units_pass_a);
    } else if (plan.mode == 2) {
        // segments, each looking back at the earlier ones and correcting itself
        e = run(kModeLookback, counters, plan.units_pass_a);
    } else {
        // segments from their own start, then the carry over segments, then
        // the start states' contributions to the outputs
        e = run(kModeSegments, counters, plan.units_pass_a);
        if (e == cudaSuccess) {
            CarryParams cp{};
            cp.A = A;
            cp.ws_h = prm.ws_h;
            cp.ws_sdt = prm.ws_sdt;
            cp.last_state = last_state;
            cp.chains = chains;
            cp.dim = dims->dim;
            cp.nseg = plan.nchunks;
            cp.dstate = (int)dims->dstate;
            const unsigned grid = (unsigned)((chains + kCarryWarps - 1) / kCarryWarps);
            if (dims->io_dtype == MAMBA_F32)
                scan_carry_kernel<true><<<grid, kCarryWarps * 32, 0, stream>>>(cp);
            else
                scan_carry_kernel<false><<<grid, kCarryWarps * 32, 0, stream>>>(cp);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess && plan.units_pass_b > 0) {
            CorrectParams q{};
            q.delta = delta;
            q.z = z;
            q.C = C;
            q.A = A;
            q.delta_bias = delta_bias;
            q.out = out;
            q.ws_h = prm.ws_h;
            q.counter = counters + 1;
            q.batch = dims->batch;
            q.dim = dims->dim;
            q.seqlen = dims->seqlen;
            q.chains = chains;
            q.seg_len = plan.chunk_len;
            q.items = plan.units_pass_b;
            q.nseg = plan.nchunks;
            q.dstate = (int)dims->dstate;
            q.bc_bf16 = dims->bc_dtype == MAMBA_BF16;
            q.vec_io = ((dims->seqlen * io_es) % 16 == 0) && aligned(delta, 16) && aligned(out, 16) &&
                       (!z || aligned(z, 16));
            q.vec_c = ((dims->seqlen * bc_es) % 16 == 0) && aligned(C, 16);
            e = dims->io_dtype == MAMBA_BF16
                    ? dispatch_correct<__nv_bfloat16>(q, has_z, sp, dev, sms, stream)
                    : dispatch_correct<float>(q, has_z, sp, dev, sms, stream);
        }
    }
    return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

extern "C" {

MAMBA_API mamba_status_t mamba_selective_state_update(float* state, const void* x, const void* dt,
                                                      const float* A, const void* B, const void* C,
                                                      const float* D, const void* z,
                                                      const float* dt_bias, void* out,
                                                      const mamba_dims_t* dims,
                                                      cudaStream_t stream) {
    mamba_status_t st = check_dims(dims, false);
    if (st != MAMBA_OK) return st;
    const int64_t chains = dims->batch * dims->dim;
    if (chains == 0) return MAMBA_OK;
    if (state == nullptr || x == nullptr || dt == nullptr || A == nullptr || B == nullptr ||
        C == nullptr || out == nullptr)
        return MAMBA_ERR_INVALID_ARG;
    const int io_es = dtype_bytes(dims->io_dtype);
    const int bc_es = dtype_bytes(dims->bc_dtype);
    if (!aligned(state, 4) || !aligned(x, io_es) || !aligned(dt, io_es) || !aligned(out, io_es) ||
        (z && !aligned(z, io_es)) || !aligned(B, bc_es) || !aligned(C, bc_es) || !aligned(A, 4) ||
        (D && !aligned(D, 4)) || (dt_bias && !aligned(dt_bias, 4)))
        return MAMBA_ERR_ALIGN;

    UpdateParams prm{};
    prm.state = state;
    prm.x = x;
    prm.dt = dt;
    prm.A = A;
    prm.B = B;
    prm.C = C;
    prm.D = D;
    prm.z = z;
    prm.dt_bias = dt_bias;
    prm.out = out;
    prm.batch = dims->batch;
    prm.dim = dims->dim;
    prm.chains = chains;
    prm.dstate = (int)dims->dstate;
    prm.dt_softplus = dims->dt_softplus != 0;
    prm.zoh = (dims->flags & MAMBA_FLAG_ZOH) != 0;
    const bool fast = dims->dstate == 16 && aligned(state, 16) && aligned(A, 16) &&
                      aligned(B, 4 * bc_es) && aligned(C, 4 * bc_es);
    // Streaming (bulk TMA) path: every bulk copy needs 16-byte aligned ends.
    const bool bulk = fast && !(dims->flags & MAMBA_FLAG_NO_TMA) && dims->dim % 8 == 0 &&
                      aligned(x, 16) && aligned(dt, 16) && aligned(out, 16) &&
                      (!z || aligned(z, 16)) && (!D || aligned(D, 16)) &&
                      (!dt_bias || aligned(dt_bias, 16)) && aligned(B, 16) && aligned(C, 16);
    const bool has_z = z != nullptr;
    const bool bc_bf16 = dims->bc_dtype == MAMBA_BF16;
    int dev = 0;
    int sms = 1;
    if (bulk) {
        sms = current_sm_count(&dev);
        if (sms <= 0) return MAMBA_ERR_CUDA;
    }
    const bool pdl = (dims->flags & MAMBA_FLAG_PDL) != 0;
    const cudaError_t e =
        dims->io_dtype == MAMBA_BF16
            ? dispatch_update<__nv_bfloat16>(prm, bc_bf16, fast, bulk, has_z, dev, sms, pdl, stream)
            : dispatch_update<float>(prm, bc_bf16, fast, bulk, has_z, dev, sms, pdl, stream);
    return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Scan without a caller workspace (mamba_selective_scan_fwd_noalloc).
//
// For callers that may not allocate device memory, the scan's scratch lives
// in this file-scope device array.  In host code `g_noalloc_scratch` names a
// host-side stand-in, not a device address: its device address is looked up
// per device with cudaGetSymbolAddress and passed to the kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MAMBA_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mutex;
void* g_noalloc_address[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) and cached.
mamba_status_t noalloc_scratch_address(void** address) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MAMBA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (dev >= 0 && dev < kMaxDevices && g_noalloc_address[dev] != nullptr) {
        *address = g_noalloc_address[dev];
        return MAMBA_OK;
    }
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
        return MAMBA_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDevices) g_noalloc_address[dev] = ptr;
    *address = ptr;
    return MAMBA_OK;
}

}  // namespace

extern "C" {

MAMBA_API mamba_status_t mamba_selective_scan_fwd_noalloc(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus, void* out,
    float* last_state, const mamba_dims_t* dims, cudaStream_t stream) {
    mamba_status_t st = check_dims(dims, true);
    if (st != MAMBA_OK) return st;
    mamba_dims_t local = *dims;
    local.workspace = nullptr;
    local.workspace_bytes = 0;
    if (local.batch * local.dim > 0 && local.seqlen > 0) {
        const int sms = current_sm_count(nullptr);
        if (sms <= 0) return MAMBA_ERR_CUDA;
        mamba_scan_plan_t plan;
        st = plan_scan(&local, sms, &plan);
        if (st != MAMBA_OK) return st;
        if (plan.workspace_bytes > MAMBA_NOALLOC_SCRATCH_BYTES) return MAMBA_ERR_TOO_LARGE;
        void* scratch = nullptr;
        st = noalloc_scratch_address(&scratch);
        if (st != MAMBA_OK) return st;
        local.workspace = scratch;
        local.workspace_bytes = MAMBA_NOALLOC_SCRATCH_BYTES;
    }
    return mamba_selective_scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus, out, last_state,
                                    &local, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Scan over host buffers (mamba_selective_scan_fwd_host): chunks of batch rows
// flow through three device stages; copies in run on one internal stream,
// scans on the caller's stream, copies out on a second internal stream.

namespace {

constexpr int kHostStages = 3;

// Device scratch of the host pipeline (offsets in bytes).
struct HostLayout {
    size_t a, d, bias;                                   // parameters, copied once
    size_t stage0, stage_bytes;                          // first stage, stage stride
    size_t u, delta, z, out, B, C, h0, last, scan;       // offsets inside a stage
    size_t scan_bytes;
    size_t total;
    int64_t rows, nchunks;
};

int64_t host_chunk_rows(const mamba_dims_t* dims, int64_t rows) {
    if (rows > 0) return std::min<int64_t>(rows, std::max<int64_t>(dims->batch, 1));
    return std::max<int64_t>(1, (dims->batch + 7) / 8);   // about 8 chunks
}

mamba_status_t host_layout(const mamba_dims_t* dims, int64_t rows_req, int sms, HostLayout* L) {
    *L = HostLayout{};
    const int64_t rows = host_chunk_rows(dims, rows_req);
    const size_t io = (size_t)dtype_bytes(dims->io_dtype), bc = (size_t)dtype_bytes(dims->bc_dtype);
    const size_t Dm = (size_t)dims->dim, N = (size_t)dims->dstate, Ls = (size_t)dims->seqlen;
    const size_t R = (size_t)rows;
    size_t off = 0;
    L->a = off;    off += align256(Dm * N * sizeof(float));
    L->d = off;    off += align256(Dm * sizeof(float));
    L->bias = off; off += align256(Dm * sizeof(float));
    L->stage0 = off;
    size_t s = 0;
    const size_t act = R * Dm * Ls * io;
    L->u = s;     s += align256(act);
    L->delta = s; s += align256(act);
    L->z = s;     s += align256(act);
    L->out = s;   s += align256(act);
    L->B = s;     s += align256(R * N * Ls * bc);
    L->C = s;     s += align256(R * N * Ls * bc);
    L->h0 = s;    s += align256(R * Dm * N * sizeof(float));
    L->last = s;  s += align256(R * Dm * N * sizeof(float));
    // Scan scratch: the larger of a full chunk's plan and the last chunk's.
    size_t scan = 0;
    const int64_t sizes[2] = {rows, dims->batch % rows};
    for (int64_t r : sizes) {
        if (r <= 0) continue;
        mamba_dims_t cd = *dims;
        cd.batch = r;
        mamba_scan_plan_t plan;
        const mamba_status_t st = plan_scan(&cd, sms, &plan);
        if (st != MAMBA_OK) return st;
        scan = std::max(scan, plan.workspace_bytes);
    }
    L->scan = s;
    s += align256(scan);
    L->scan_bytes = scan;
    L->stage_bytes = s;
    L->total = off + kHostStages * s;
    L->rows = rows;
    L->nchunks = (dims->batch + rows - 1) / rows;
    return MAMBA_OK;
}

// Copy streams and events of the host pipeline, created once per device.
struct HostPipe {
    cudaStream_t h2d = nullptr;
    cudaStream_t d2h = nullptr;
    cudaEvent_t start = nullptr;
    cudaEvent_t h2d_done[kHostStages] = {};
    cudaEvent_t comp_done[kHostStages] = {};
    cudaEvent_t d2h_done[kHostStages] = {};
    bool ready = false;
};

std::mutex g_host_mutex;          // held while a call enqueues its work
HostPipe g_host_pipe[kMaxDevices];

// Called with g_host_mutex held and the device current.
mamba_status_t host_pipe(int dev, HostPipe** out) {
    if (dev < 0 || dev >= kMaxDevices) return MAMBA_ERR_CUDA;
    HostPipe& p = g_host_pipe[dev];
    if (!p.ready) {
        HostPipe q;
        bool ok = cudaStreamCreateWithFlags(&q.h2d, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&q.d2h, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaEventCreateWithFlags(&q.start, cudaEventDisableTiming) == cudaSuccess;
        for (int i = 0; ok && i < kHostStages; ++i)
            ok = cudaEventCreateWithFlags(&q.h2d_done[i], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&q.comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&q.d2h_done[i], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) return MAMBA_ERR_CUDA;   // handles made so far are kept by the runtime until exit
        q.ready = true;
        p = q;
    }
    *out = &p;
    return MAMBA_OK;
}

cudaError_t copy_async(void* dst, const void* src, size_t bytes, cudaMemcpyKind kind,
                       cudaStream_t stream) {
    if (bytes == 0 || src == nullptr || dst == nullptr) return cudaSuccess;
    return cudaMemcpyAsync(dst, src, bytes, kind, stream);
}

}  // namespace

extern "C" {

MAMBA_API size_t mamba_selective_scan_host_workspace_bytes(const mamba_dims_t* dims, int64_t rows) {
    if (check_dims(dims, true) != MAMBA_OK || rows < 0) return static_cast<size_t>(-1);
    if (dims->batch * dims->dim == 0) return 0;
    const int sms = current_sm_count(nullptr);
    if (sms <= 0) return static_cast<size_t>(-1);
    HostLayout L;
    if (host_layout(dims, rows, sms, &L) != MAMBA_OK) return static_cast<size_t>(-1);
    return L.total;
}

MAMBA_API mamba_status_t mamba_selective_scan_fwd_host(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus,
    const float* initial_state, void* out, float* last_state, int64_t rows,
    const mamba_dims_t* dims, cudaStream_t stream) {
    mamba_status_t st = check_dims(dims, true);
    if (st != MAMBA_OK) return st;
    if (rows < 0) return MAMBA_ERR_INVALID_ARG;
    const int64_t chains = dims->batch * dims->dim;
    if (chains == 0) return MAMBA_OK;
    if (A == nullptr) return MAMBA_ERR_INVALID_ARG;
    if (dims->seqlen > 0 &&
        (u == nullptr || delta == nullptr || B == nullptr || C == nullptr || out == nullptr))
        return MAMBA_ERR_INVALID_ARG;
    const size_t state_bytes = (size_t)chains * dims->dstate * sizeof(float);
    if (initial_state != nullptr && last_state != nullptr && initial_state != last_state) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(initial_state);
        const uintptr_t b = reinterpret_cast<uintptr_t>(last_state);
        if (a < b + state_bytes && b < a + state_bytes) return MAMBA_ERR_INVALID_ARG;
    }
    int dev = 0;
    const int sms = current_sm_count(&dev);
    if (sms <= 0) return MAMBA_ERR_CUDA;
    HostLayout L;
    st = host_layout(dims, rows, sms, &L);
    if (st != MAMBA_OK) return st;
    if (dims->workspace == nullptr || dims->workspace_bytes < L.total) return MAMBA_ERR_WORKSPACE;
    if (!aligned(dims->workspace, 256)) return MAMBA_ERR_ALIGN;

    std::lock_guard<std::mutex> lock(g_host_mutex);
    HostPipe* pp = nullptr;
    st = host_pipe(dev, &pp);
    if (st != MAMBA_OK) return st;
    uint8_t* ws = static_cast<uint8_t*>(dims->workspace);
    const size_t io = (size_t)dtype_bytes(dims->io_dtype), bc = (size_t)dtype_bytes(dims->bc_dtype);
    const size_t Dm = (size_t)dims->dim, N = (size_t)dims->dstate, Ls = (size_t)dims->seqlen;
    float* dA = reinterpret_cast<float*>(ws + L.a);
    float* dD = D ? reinterpret_cast<float*>(ws + L.d) : nullptr;
    float* dbias = delta_bias ? reinterpret_cast<float*>(ws + L.bias) : nullptr;
    auto fail = [](cudaError_t e) { return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA; };

    // Parameters, on the scan stream ahead of every chunk.
    cudaError_t e = copy_async(dA, A, Dm * N * sizeof(float), cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = copy_async(dD, D, Dm * sizeof(float), cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess)
        e = copy_async(dbias, delta_bias, Dm * sizeof(float), cudaMemcpyHostToDevice, stream);
    // Both copy streams start after the earlier work on `stream`.
    if (e == cudaSuccess) e = cudaEventRecord(pp->start, stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(pp->h2d, pp->start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(pp->d2h, pp->start, 0);
    if (e != cudaSuccess) return MAMBA_ERR_CUDA;

    const uint8_t* hu = static_cast<const uint8_t*>(u);
    const uint8_t* hdelta = static_cast<const uint8_t*>(delta);
    const uint8_t* hz = static_cast<const uint8_t*>(z);
    const uint8_t* hB = static_cast<const uint8_t*>(B);
    const uint8_t* hC = static_cast<const uint8_t*>(C);
    uint8_t* hout = static_cast<uint8_t*>(out);
    for (int64_t c = 0; c < L.nchunks; ++c) {
        const int s = (int)(c % kHostStages);
        const size_t b0 = (size_t)(c * L.rows);
        const size_t r = (size_t)std::min<int64_t>(L.rows, dims->batch - (int64_t)b0);
        uint8_t* stg = ws + L.stage0 + (size_t)s * L.stage_bytes;
        const size_t act = r * Dm * Ls * io, act0 = b0 * Dm * Ls * io;
        const size_t bcb = r * N * Ls * bc, bc0 = b0 * N * Ls * bc;
        const size_t sb = r * Dm * N * sizeof(float), s0 = b0 * Dm * N;
        // in: stage s is free once the scan of chunk c - 3 has read it
        if (c >= kHostStages) e = cudaStreamWaitEvent(pp->h2d, pp->comp_done[s], 0);
        if (e == cudaSuccess) e = copy_async(stg + L.u, hu ? hu + act0 : nullptr, act, cudaMemcpyHostToDevice, pp->h2d);
        if (e == cudaSuccess) e = copy_async(stg + L.delta, hdelta ? hdelta + act0 : nullptr, act, cudaMemcpyHostToDevice, pp->h2d);
        if (e == cudaSuccess) e = copy_async(stg + L.z, hz ? hz + act0 : nullptr, act, cudaMemcpyHostToDevice, pp->h2d);
        if (e == cudaSuccess) e = copy_async(stg + L.B, hB ? hB + bc0 : nullptr, bcb, cudaMemcpyHostToDevice, pp->h2d);
        if (e == cudaSuccess) e = copy_async(stg + L.C, hC ? hC + bc0 : nullptr, bcb, cudaMemcpyHostToDevice, pp->h2d);
        if (e == cudaSuccess)
            e = copy_async(stg + L.h0, initial_state ? initial_state + s0 : nullptr, sb, cudaMemcpyHostToDevice, pp->h2d);
        if (e == cudaSuccess) e = cudaEventRecord(pp->h2d_done[s], pp->h2d);
        // scan: after its inputs, and after chunk c - 3's outputs left stage s
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, pp->h2d_done[s], 0);
        if (e == cudaSuccess && c >= kHostStages) e = cudaStreamWaitEvent(stream, pp->d2h_done[s], 0);
        if (e != cudaSuccess) return MAMBA_ERR_CUDA;
        mamba_dims_t cd = *dims;
        cd.batch = (int64_t)r;
        cd.workspace = stg + L.scan;
        cd.workspace_bytes = L.scan_bytes;
        st = mamba_selective_scan_fwd_with_state(
            stg + L.u, stg + L.delta, dA, stg + L.B, stg + L.C, dD, z ? stg + L.z : nullptr, dbias,
            softplus, initial_state ? reinterpret_cast<float*>(stg + L.h0) : nullptr, stg + L.out,
            last_state ? reinterpret_cast<float*>(stg + L.last) : nullptr, &cd, stream);
        if (st != MAMBA_OK) return st;
        e = cudaEventRecord(pp->comp_done[s], stream);
        // out: after the scan of chunk c
        if (e == cudaSuccess) e = cudaStreamWaitEvent(pp->d2h, pp->comp_done[s], 0);
        if (e == cudaSuccess) e = copy_async(hout ? hout + act0 : nullptr, stg + L.out, act, cudaMemcpyDeviceToHost, pp->d2h);
        if (e == cudaSuccess)
            e = copy_async(last_state ? last_state + s0 : nullptr, stg + L.last, last_state ? sb : 0,
                           cudaMemcpyDeviceToHost, pp->d2h);
        if (e == cudaSuccess) e = cudaEventRecord(pp->d2h_done[s], pp->d2h);
        if (e != cudaSuccess) return MAMBA_ERR_CUDA;
    }
    // Later work on `stream` follows the last copy back (the copy-in stream
    // already joined it through the scans' waits).
    return fail(cudaStreamWaitEvent(stream, pp->d2h_done[(L.nchunks - 1) % kHostStages], 0));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Short causal convolution (prefill and decode update).

namespace {

mamba_status_t check_conv(const mamba_dims_t* dims, int width, bool seq) {
    if (dims == nullptr) return MAMBA_ERR_INVALID_ARG;
    if (dims->batch < 0 || dims->dim < 0 || (seq && dims->seqlen < 0)) return MAMBA_ERR_INVALID_ARG;
    if (width < 1 || width > MAMBA_MAX_CONV_WIDTH) return MAMBA_ERR_UNSUPPORTED;
    if (!dtype_ok(dims->io_dtype)) return MAMBA_ERR_UNSUPPORTED;
    const int64_t lim = (int64_t)1 << 40;
    if (dims->batch >= lim || dims->dim >= lim || (seq && dims->seqlen >= lim))
        return MAMBA_ERR_INVALID_ARG;
    return MAMBA_OK;
}

bool partly_overlap(const void* a, const void* b, size_t bytes) {
    if (a == nullptr || b == nullptr || a == b) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + bytes && y < x + bytes;
}

unsigned int blocks_for(int64_t threads) {
    return (unsigned int)((threads + kConvThreads - 1) / kConvThreads);
}

template <typename IoT>
cudaError_t launch_conv_fwd(const ConvParams& prm, bool vec, cudaStream_t stream) {
    if (prm.seqlen > 0) {
        if (vec) {
            const int64_t warps = prm.chains * ((prm.vec_per_row + 32 * kConvVecs - 1) / (32 * kConvVecs));
            const unsigned int grid = blocks_for(warps * 32);
            switch (prm.width) {
                case 1: causal_conv1d_vec_kernel<IoT, 1><<<grid, kConvThreads, 0, stream>>>(prm); break;
                case 2: causal_conv1d_vec_kernel<IoT, 2><<<grid, kConvThreads, 0, stream>>>(prm); break;
                case 3: causal_conv1d_vec_kernel<IoT, 3><<<grid, kConvThreads, 0, stream>>>(prm); break;
                default: causal_conv1d_vec_kernel<IoT, 4><<<grid, kConvThreads, 0, stream>>>(prm); break;
            }
        } else {
            causal_conv1d_generic_kernel<IoT><<<blocks_for(prm.chains * prm.seqlen), kConvThreads, 0,
                                               stream>>>(prm);
        }
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (prm.final_state != nullptr)
        causal_conv1d_final_state_kernel<IoT><<<blocks_for(prm.chains), kConvThreads, 0, stream>>>(prm);
    return cudaGetLastError();
}

}  // namespace

extern "C" {

MAMBA_API mamba_status_t mamba_causal_conv1d_fwd(const void* x, const float* weight,
                                                 const float* bias, const void* initial_conv_state,
                                                 int width, int silu, void* out,
                                                 void* final_conv_state, const mamba_dims_t* dims,
                                                 cudaStream_t stream) {
    mamba_status_t st = check_conv(dims, width, true);
    if (st != MAMBA_OK) return st;
    const int64_t chains = dims->batch * dims->dim;
    if (chains == 0) return MAMBA_OK;
    if (weight == nullptr) return MAMBA_ERR_INVALID_ARG;
    if (dims->seqlen > 0 && (x == nullptr || out == nullptr)) return MAMBA_ERR_INVALID_ARG;
    const int es = dtype_bytes(dims->io_dtype);
    if ((x && !aligned(x, es)) || (out && !aligned(out, es)) || !aligned(weight, 4) ||
        (bias && !aligned(bias, 4)) || (initial_conv_state && !aligned(initial_conv_state, es)) ||
        (final_conv_state && !aligned(final_conv_state, es)))
        return MAMBA_ERR_ALIGN;
    if (partly_overlap(initial_conv_state, final_conv_state, (size_t)chains * width * es))
        return MAMBA_ERR_INVALID_ARG;
    if (dims->seqlen > 0 && x == out) return MAMBA_ERR_INVALID_ARG;
    if (chains * std::max<int64_t>(dims->seqlen, 1) / kConvThreads >= ((int64_t)1 << 31))
        return MAMBA_ERR_UNSUPPORTED;
    ConvParams prm{};
    prm.x = x;
    prm.weight = weight;
    prm.bias = bias;
    prm.init = initial_conv_state;
    prm.out = out;
    prm.final_state = final_conv_state;
    prm.batch = dims->batch;
    prm.dim = dims->dim;
    prm.seqlen = dims->seqlen;
    prm.chains = chains;
    prm.width = width;
    prm.silu = silu != 0;
    const bool vec = (dims->seqlen * es) % 16 == 0 && aligned(x, 16) && aligned(out, 16);
    prm.vec_per_row = vec ? dims->seqlen * es / 16 : 0;
    const cudaError_t e = dims->io_dtype == MAMBA_BF16
                              ? launch_conv_fwd<__nv_bfloat16>(prm, vec, stream)
                              : launch_conv_fwd<float>(prm, vec, stream);
    return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

MAMBA_API mamba_status_t mamba_causal_conv1d_update(void* conv_state, const void* x,
                                                    const float* weight, const float* bias,
                                                    int width, int silu, void* out,
                                                    const mamba_dims_t* dims,
                                                    cudaStream_t stream) {
    mamba_status_t st = check_conv(dims, width, false);
    if (st != MAMBA_OK) return st;
    const int64_t chains = dims->batch * dims->dim;
    if (chains == 0) return MAMBA_OK;
    if (conv_state == nullptr || x == nullptr || weight == nullptr || out == nullptr)
        return MAMBA_ERR_INVALID_ARG;
    const int es = dtype_bytes(dims->io_dtype);
    if (!aligned(conv_state, es) || !aligned(x, es) || !aligned(out, es) || !aligned(weight, 4) ||
        (bias && !aligned(bias, 4)))
        return MAMBA_ERR_ALIGN;
    if (chains / kConvThreads >= ((int64_t)1 << 31)) return MAMBA_ERR_UNSUPPORTED;
    ConvParams prm{};
    prm.x = x;
    prm.weight = weight;
    prm.bias = bias;
    prm.state = conv_state;
    prm.out = out;
    prm.batch = dims->batch;
    prm.dim = dims->dim;
    prm.chains = chains;
    prm.width = width;
    prm.silu = silu != 0;
    // W = 4: kConvUpdateChains chains per thread when the state is aligned to its
    // vector and x/out to that many elements, else one chain per thread.
    constexpr int kC = kConvUpdateChains;
    const bool w4xn = width == 4 && aligned(conv_state, 4 * es) && aligned(x, kC * es) &&
                      aligned(out, kC * es) && aligned(weight, 16);
    const bool w4 = width == 4 && aligned(conv_state, 4 * es) && aligned(weight, 16);
    const unsigned int grid = blocks_for(w4xn ? (chains + kC - 1) / kC : chains);
    // MAMBA_FLAG_PDL: the vector path as a programmatic dependent launch (the
    // other paths ignore the flag).
    const bool pdl = w4xn && (dims->flags & MAMBA_FLAG_PDL) != 0;
    if (pdl) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kConvThreads);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t e =
            dims->io_dtype == MAMBA_BF16
                ? cudaLaunchKernelEx(&cfg, causal_conv1d_update_w4xn_kernel<__nv_bfloat16, kC, true>, prm)
                : cudaLaunchKernelEx(&cfg, causal_conv1d_update_w4xn_kernel<float, kC, true>, prm);
        if (e != cudaSuccess) return MAMBA_ERR_CUDA;
    } else if (dims->io_dtype == MAMBA_BF16) {
        if (w4xn) causal_conv1d_update_w4xn_kernel<__nv_bfloat16, kC, false><<<grid, kConvThreads, 0, stream>>>(prm);
        else if (w4) causal_conv1d_update_w4_kernel<__nv_bfloat16><<<grid, kConvThreads, 0, stream>>>(prm);
        else causal_conv1d_update_kernel<__nv_bfloat16><<<grid, kConvThreads, 0, stream>>>(prm);
    } else {
        if (w4xn) causal_conv1d_update_w4xn_kernel<float, kC, false><<<grid, kConvThreads, 0, stream>>>(prm);
        else if (w4) causal_conv1d_update_w4_kernel<float><<<grid, kConvThreads, 0, stream>>>(prm);
        else causal_conv1d_update_kernel<float><<<grid, kConvThreads, 0, stream>>>(prm);
    }
    return cudaGetLastError() == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward pass of the scan.

namespace {

// Scratch of one backward call (offsets in bytes).
struct BwdWorkspace {
    size_t fwd_zeroed;      // checkpoint pass: counters + flags, cleared
    size_t fwd_bytes;       // checkpoint pass scratch (zeroed part + carry)
    size_t bwd;             // backward: counter at +0, flags at +kWsFlags
    size_t bwd_zeroed;
    size_t bwd_carry;       // [chains][16] lambda handoff
    size_t ckpt;            // [chains][tiles][16] fp32
    size_t total;
    int64_t K, seg_len, groups, tiles;
};

// Segments of the backward (chained, in reverse): the chained rule of the
// forward planner, K = min(ceil(8 W / G), L / 256), at least 1.
mamba_status_t bwd_layout(const mamba_dims_t* dims, int sms, BwdWorkspace* w) {
    *w = BwdWorkspace{};
    const int io_es = dtype_bytes(dims->io_dtype);
    const int64_t T = kRowBytes / io_es;                   // forward tile, a multiple of 8
    const int64_t L = dims->seqlen;
    const int64_t groups = dims->batch * ((dims->dim + 31) / 32);
    const int64_t W = (int64_t)sms * ScanLayout<1>::kWarpsPerSm;
    int64_t K = 1;
    if (groups > 0 && L > 0) K = std::max<int64_t>(1, std::min<int64_t>((8 * W + groups - 1) / groups, L / 256));
    int64_t seg = L;
    if (K > 1) {
        seg = ((L + K - 1) / K + T - 1) / T * T;
        K = (L + seg - 1) / seg;
    }
    if (K <= 1) { K = 1; seg = L; }
    if (groups * K >= ((int64_t)1 << 31)) return MAMBA_ERR_UNSUPPORTED;
    const size_t chains = (size_t)dims->batch * (size_t)dims->dim;
    const int64_t tiles = (L + kCkptSteps - 1) / kCkptSteps;
    size_t off = 0;
    w->fwd_zeroed = kWsFlags + align256((size_t)groups * sizeof(unsigned int));
    off = w->fwd_zeroed + (K > 1 ? align256(chains * kNPad * sizeof(float)) : 0);
    w->fwd_bytes = off;
    w->bwd = off;
    w->bwd_zeroed = kWsFlags + align256((size_t)groups * sizeof(unsigned int));
    off += w->bwd_zeroed;
    w->bwd_carry = off;
    off += align256(chains * kNPad * sizeof(float));
    w->ckpt = off;
    off += align256(chains * (size_t)tiles * kNPad * sizeof(float));
    w->total = off;
    w->K = K;
    w->seg_len = seg;
    w->groups = groups;
    w->tiles = tiles;
    return MAMBA_OK;
}

template <typename IoT, typename BcT, bool kHasZ, bool kZoh, bool kBld>
cudaError_t launch_bwd(const BwdParams& prm, int dev, int sms, cudaStream_t stream) {
    static bool attr_done[kMaxDevices] = {false};
    static int resident[kMaxDevices] = {0};
    auto kernel = selective_scan_bwd_kernel<IoT, BcT, kHasZ, kZoh, kBld>;
    constexpr int smem = kBwdWarps * bwd_warp_smem<IoT, BcT>();
    cudaError_t e = ensure_smem_attr(kernel, smem, attr_done, dev);
    if (e != cudaSuccess) return e;
    int per_sm = (dev >= 0 && dev < kMaxDevices) ? resident[dev] : 0;
    if (per_sm <= 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kBwdWarps * 32, smem);
        if (e != cudaSuccess) return e;
        if (per_sm <= 0) return cudaErrorInvalidConfiguration;
        if (dev >= 0 && dev < kMaxDevices) resident[dev] = per_sm;
    }
    // At most one segment per group can run at a time (the chain of segments).
    const int64_t want = (std::min<int64_t>(prm.items, prm.groups) + kBwdWarps - 1) / kBwdWarps;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)per_sm * sms));
    kernel<<<(unsigned)grid, kBwdWarps * 32, smem, stream>>>(prm);
    return cudaGetLastError();
}

template <typename IoT, bool kZoh, bool kBld>
cudaError_t dispatch_bwd_zoh(const BwdParams& prm, bool has_z, int dev, int sms, cudaStream_t stream) {
    if (prm.bc_bf16)
        return has_z ? launch_bwd<IoT, __nv_bfloat16, true, kZoh, kBld>(prm, dev, sms, stream)
                     : launch_bwd<IoT, __nv_bfloat16, false, kZoh, kBld>(prm, dev, sms, stream);
    return has_z ? launch_bwd<IoT, float, true, kZoh, kBld>(prm, dev, sms, stream)
                 : launch_bwd<IoT, float, false, kZoh, kBld>(prm, dev, sms, stream);
}

// Kernel instance for (zero-order hold, activation layout).
template <typename IoT>
cudaError_t dispatch_bwd(const BwdParams& prm, bool has_z, bool zoh, bool bld, int dev, int sms,
                         cudaStream_t stream) {
    if (bld)
        return zoh ? dispatch_bwd_zoh<IoT, true, true>(prm, has_z, dev, sms, stream)
                   : dispatch_bwd_zoh<IoT, false, true>(prm, has_z, dev, sms, stream);
    return zoh ? dispatch_bwd_zoh<IoT, true, false>(prm, has_z, dev, sms, stream)
               : dispatch_bwd_zoh<IoT, false, false>(prm, has_z, dev, sms, stream);
}

cudaError_t zero_async(void* p, size_t bytes, cudaStream_t stream) {
    return (p == nullptr || bytes == 0) ? cudaSuccess : cudaMemsetAsync(p, 0, bytes, stream);
}

}  // namespace

namespace {

// Map over a row-major bf16 (batch, L, heads_or_groups, width) tensor whose one
// box is a whole 128-row operand tile of the Mamba-2 layer kernel in its
// shared-memory layout: dimensions (64 elements, L, width / 64 column halves,
// heads_or_groups, batch), box (64, 128, width / 64, 1, 1), 128-byte swizzle,
// so that shared memory receives each 64-column half as 128 rows of 128 bytes
// in 1024-byte swizzle atoms, halves 16 KB apart.
bool encode_map_ssd(CUtensorMap* map, const void* base, uint64_t width, uint64_t heads,
                    uint64_t L, uint64_t batch) {
    auto encode = tensor_map_encoder();
    if (encode == nullptr) return false;
    const uint64_t row = heads * width * 2;                 // bytes between tokens
    const cuuint64_t dims[5] = {64, L, width / 64, heads, batch};
    const cuuint64_t strides[4] = {row, 128, width * 2, row * L};
    const cuuint32_t box[5] = {64, (cuuint32_t)kSsdQ, (cuuint32_t)(width / 64), 1, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Argument checks of the Mamba-2 layer; MAMBA_OK when a launch may follow.
mamba_status_t check_ssd(const void* x, const void* dt, const float* A, const void* B,
                         const void* C, const float* D, const void* z, const float* dt_bias,
                         const float* initial_state, const void* out, const float* final_state,
                         const mamba_ssd_dims_t* d) {
    if (d == nullptr) return MAMBA_ERR_INVALID_ARG;
    if (d->batch < 0 || d->seqlen < 0 || d->nheads < 1 || d->ngroups < 1 || d->headdim < 1 ||
        d->dstate < 1)
        return MAMBA_ERR_INVALID_ARG;
    if (d->nheads % d->ngroups != 0) return MAMBA_ERR_INVALID_ARG;
    if (d->headdim != kSsdP || d->dstate != kSsdN || d->io_dtype != MAMBA_BF16)
        return MAMBA_ERR_UNSUPPORTED;
    const int64_t lim = (int64_t)1 << 31;
    if (d->batch * d->nheads >= lim || d->seqlen >= lim) return MAMBA_ERR_INVALID_ARG;
    if (A == nullptr) return MAMBA_ERR_INVALID_ARG;
    if (d->batch > 0 && d->seqlen > 0 &&
        (x == nullptr || dt == nullptr || B == nullptr || C == nullptr || out == nullptr))
        return MAMBA_ERR_INVALID_ARG;
    if ((x && !aligned(x, 16)) || (z && !aligned(z, 16)) || (out && !aligned(out, 16)) ||
        (B && !aligned(B, 16)) || (C && !aligned(C, 16)) || (dt && !aligned(dt, 2)) ||
        !aligned(A, 4) || (D && !aligned(D, 4)) || (dt_bias && !aligned(dt_bias, 4)) ||
        (initial_state && !aligned(initial_state, 4)) || (final_state && !aligned(final_state, 4)))
        return MAMBA_ERR_ALIGN;
    return MAMBA_OK;
}

}  // namespace

extern "C" {

MAMBA_API mamba_status_t mamba_ssd_chunk_scan_fwd(const void* x, const void* dt, const float* A,
                                                  const void* B, const void* C, const float* D,
                                                  const void* z, const float* dt_bias,
                                                  const float* initial_state, void* out,
                                                  float* final_state,
                                                  const mamba_ssd_dims_t* dims,
                                                  cudaStream_t stream) {
    const mamba_status_t st = check_ssd(x, dt, A, B, C, D, z, dt_bias, initial_state, out,
                                        final_state, dims);
    if (st != MAMBA_OK) return st;
    if (dims->batch == 0) return MAMBA_OK;
    if (dims->seqlen == 0 && final_state == nullptr) return MAMBA_OK;
    int dev = 0;
    if (current_sm_count(&dev) <= 0) return MAMBA_ERR_CUDA;
    static bool attr_done[kMaxDevices] = {false};
    cudaError_t e = ensure_smem_attr(ssd_chunk_scan_kernel, kSsdSmemBytes, attr_done, dev);
    if (e != cudaSuccess) return MAMBA_ERR_CUDA;
    SsdParams prm;
    prm.x = static_cast<const __nv_bfloat16*>(x);
    prm.dt = static_cast<const __nv_bfloat16*>(dt);
    prm.A = A;
    prm.B = static_cast<const __nv_bfloat16*>(B);
    prm.C = static_cast<const __nv_bfloat16*>(C);
    prm.D = D;
    prm.z = static_cast<const __nv_bfloat16*>(z);
    prm.dt_bias = dt_bias;
    prm.h0 = initial_state;
    prm.out = static_cast<__nv_bfloat16*>(out);
    prm.hT = final_state;
    prm.seqlen = dims->seqlen;
    prm.nheads = (int)dims->nheads;
    prm.ngroups = (int)dims->ngroups;
    prm.softplus = dims->dt_softplus != 0;
    // TMA maps over x, z, out (batch, L, nheads, 64) and B, C (batch, L, ngroups,
    // 128).  With L == 0 no chunk runs and the maps are never read.
    CUtensorMap maps[5];
    std::memset(maps, 0, sizeof(maps));
    if (dims->seqlen > 0) {
        const uint64_t Bt = (uint64_t)dims->batch, L = (uint64_t)dims->seqlen;
        const uint64_t H = (uint64_t)dims->nheads, G = (uint64_t)dims->ngroups;
        const bool ok = encode_map_ssd(&maps[0], x, kSsdP, H, L, Bt) &&
                        encode_map_ssd(&maps[1], z ? z : x, kSsdP, H, L, Bt) &&
                        encode_map_ssd(&maps[2], B, kSsdN, G, L, Bt) &&
                        encode_map_ssd(&maps[3], C, kSsdN, G, L, Bt) &&
                        encode_map_ssd(&maps[4], out, kSsdP, H, L, Bt);
        // (each map: one box per 128-row tile)
        if (!ok) return MAMBA_ERR_CUDA;
    }
    const unsigned grid = (unsigned)(dims->batch * dims->nheads);
    ssd_chunk_scan_kernel<<<grid, kSsdThreads, kSsdSmemBytes, stream>>>(prm, maps[0], maps[1],
                                                                        maps[2], maps[3], maps[4]);
    e = cudaGetLastError();
    return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

}  // extern "C"

extern "C" {

MAMBA_API size_t mamba_selective_scan_bwd_workspace_bytes(const mamba_dims_t* dims) {
    if (check_dims(dims, true) != MAMBA_OK) return static_cast<size_t>(-1);
    if (dims->batch * dims->dim == 0 || dims->seqlen == 0) return 0;
    const int sms = current_sm_count(nullptr);
    if (sms <= 0) return static_cast<size_t>(-1);
    BwdWorkspace w;
    if (bwd_layout(dims, sms, &w) != MAMBA_OK) return static_cast<size_t>(-1);
    return w.total;
}

MAMBA_API mamba_status_t mamba_selective_scan_bwd(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus,
    const float* initial_state, const void* dout, const float* dlast_state, void* du,
    void* ddelta, float* dA, float* dB, float* dC, float* dD, void* dz, float* ddelta_bias,
    float* dinitial_state, const mamba_dims_t* dims, cudaStream_t stream) {
    mamba_status_t st = check_dims(dims, true);
    if (st != MAMBA_OK) return st;
    const bool bld = (dims->flags & MAMBA_FLAG_LAYOUT_BLD) != 0;
    const int64_t chains = dims->batch * dims->dim;
    if (chains == 0) return MAMBA_OK;
    const int64_t L = dims->seqlen, N = dims->dstate;
    if (A == nullptr || dA == nullptr) return MAMBA_ERR_INVALID_ARG;
    if (L > 0 && (u == nullptr || delta == nullptr || B == nullptr || C == nullptr ||
                  dout == nullptr || du == nullptr || ddelta == nullptr || dB == nullptr ||
                  dC == nullptr))
        return MAMBA_ERR_INVALID_ARG;
    const int io_es = dtype_bytes(dims->io_dtype);
    const int bc_es = dtype_bytes(dims->bc_dtype);
    const void* io_ptrs[7] = {u, delta, z, dout, du, ddelta, dz};
    for (const void* q : io_ptrs)
        if (q && !aligned(q, io_es)) return MAMBA_ERR_ALIGN;
    const void* f32_ptrs[10] = {A, D, delta_bias, initial_state, dlast_state, dA, dD,
                                ddelta_bias, dinitial_state, nullptr};
    for (const void* q : f32_ptrs)
        if (q && !aligned(q, 4)) return MAMBA_ERR_ALIGN;
    if ((B && !aligned(B, bc_es)) || (C && !aligned(C, bc_es)) || (dB && !aligned(dB, 4)) ||
        (dC && !aligned(dC, 4)))
        return MAMBA_ERR_ALIGN;
    cudaError_t e = cudaSuccess;
    // gradients that are sums start from zero
    e = zero_async(dA, (size_t)dims->dim * N * sizeof(float), stream);
    if (e == cudaSuccess) e = zero_async(dD, (size_t)dims->dim * sizeof(float), stream);
    if (e == cudaSuccess) e = zero_async(ddelta_bias, (size_t)dims->dim * sizeof(float), stream);
    if (e != cudaSuccess) return MAMBA_ERR_CUDA;
    if (L == 0) {       // nothing to scan: the start state's gradient is dlast_state
        const size_t sb = (size_t)chains * N * sizeof(float);
        if (dinitial_state == nullptr) return MAMBA_OK;
        e = dlast_state ? cudaMemcpyAsync(dinitial_state, dlast_state, sb, cudaMemcpyDeviceToDevice, stream)
                        : cudaMemsetAsync(dinitial_state, 0, sb, stream);
        return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
    }
    int dev = 0;
    const int sms = current_sm_count(&dev);
    if (sms <= 0) return MAMBA_ERR_CUDA;
    BwdWorkspace w;
    st = bwd_layout(dims, sms, &w);
    if (st != MAMBA_OK) return st;
    if (dims->workspace == nullptr || dims->workspace_bytes < w.total) return MAMBA_ERR_WORKSPACE;
    if (!aligned(dims->workspace, 256)) return MAMBA_ERR_ALIGN;
    uint8_t* ws = static_cast<uint8_t*>(dims->workspace);
    e = zero_async(dB, (size_t)dims->batch * N * L * sizeof(float), stream);
    if (e == cudaSuccess) e = zero_async(dC, (size_t)dims->batch * N * L * sizeof(float), stream);
    if (e == cudaSuccess) e = zero_async(ws + w.bwd, w.bwd_zeroed, stream);
    if (e != cudaSuccess) return MAMBA_ERR_CUDA;

    // 1. checkpoint pass: the forward, chained in w.K segments, states only
    mamba_dims_t fd = *dims;
    fd.num_chunks = (int32_t)w.K;
    fd.flags = (dims->flags & (MAMBA_FLAG_NO_TMA | MAMBA_FLAG_ZOH | MAMBA_FLAG_LAYOUT_BLD)) |
               MAMBA_FLAG_ONE_LANE_PER_CHANNEL;
    fd.workspace = ws;
    fd.workspace_bytes = w.fwd_bytes;
    float* ckpt = reinterpret_cast<float*>(ws + w.ckpt);
    st = scan_fwd_internal(u, delta, A, B, C, nullptr, nullptr, delta_bias, softplus,
                           initial_state, nullptr, nullptr, &fd, stream, ckpt, w.tiles);
    if (st != MAMBA_OK) return st;

    // 2. the adjoint, segments in reverse
    BwdParams prm{};
    prm.u = u;
    prm.delta = delta;
    prm.z = z;
    prm.dout = dout;
    prm.A = A;
    prm.B = B;
    prm.C = C;
    prm.D = D;
    prm.delta_bias = delta_bias;
    prm.dlast = dlast_state;
    prm.ckpt = ckpt;
    prm.du = du;
    prm.ddelta = ddelta;
    prm.dz = dz;
    prm.dA = dA;
    prm.dB = dB;
    prm.dC = dC;
    prm.dD = dD;
    prm.dbias = ddelta_bias;
    prm.dh0 = dinitial_state;
    prm.counter = reinterpret_cast<unsigned int*>(ws + w.bwd + kWsCounters);
    prm.flags = reinterpret_cast<unsigned int*>(ws + w.bwd + kWsFlags);
    prm.carry = reinterpret_cast<float*>(ws + w.bwd_carry);
    prm.batch = dims->batch;
    prm.dim = dims->dim;
    prm.seqlen = L;
    prm.groups_per_batch = (dims->dim + 31) / 32;
    prm.groups = w.groups;
    prm.chains = chains;
    prm.seg_len = w.seg_len;
    prm.items = w.groups * w.K;
    prm.ckpt_tiles = w.tiles;
    prm.dstate = (int)N;
    prm.nseg = (int)w.K;
    prm.softplus = softplus != 0;
    prm.bc_bf16 = dims->bc_dtype == MAMBA_BF16;
    bool vec = true;
    for (const void* q : io_ptrs)
        if (q && !aligned(q, 16)) vec = false;
    prm.vec_ok = vec ? 1 : 0;
    prm.bld = bld ? 1 : 0;
    prm.bc_vec = ((L * bc_es) % 16 == 0 && aligned(B, 16) && aligned(C, 16)) ? 1 : 0;
    prm.flag_poll_limit =
        (unsigned int)std::min<int64_t>(std::max<int64_t>(w.seg_len * 256, 1 << 20), (int64_t)1 << 31);
    const bool zoh = (dims->flags & MAMBA_FLAG_ZOH) != 0;
    e = dims->io_dtype == MAMBA_BF16
            ? dispatch_bwd<__nv_bfloat16>(prm, z != nullptr, zoh, bld, dev, sms, stream)
            : dispatch_bwd<float>(prm, z != nullptr, zoh, bld, dev, sms, stream);
    return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

MAMBA_API mamba_status_t mamba_device_status(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return MAMBA_ERR_CUDA;
    int code = 0;
    if (cudaMemcpyFromSymbol(&code, g_device_status, sizeof(int)) != cudaSuccess)
        return MAMBA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess)
        return MAMBA_ERR_CUDA;
    return static_cast<mamba_status_t>(code);
}

MAMBA_API const char* mamba_status_string(mamba_status_t status) {
    switch (status) {
        case MAMBA_OK: return "MAMBA_OK";
        case MAMBA_ERR_INVALID_ARG: return "MAMBA_ERR_INVALID_ARG";
        case MAMBA_ERR_UNSUPPORTED: return "MAMBA_ERR_UNSUPPORTED";
        case MAMBA_ERR_ALIGN: return "MAMBA_ERR_ALIGN";
        case MAMBA_ERR_WORKSPACE: return "MAMBA_ERR_WORKSPACE";
        case MAMBA_ERR_CUDA: return "MAMBA_ERR_CUDA";
        case MAMBA_ERR_TIMEOUT: return "MAMBA_ERR_TIMEOUT";
        case MAMBA_ERR_TOO_LARGE: return "MAMBA_ERR_TOO_LARGE";
    }
    return "MAMBA_ERR_UNKNOWN";
}

MAMBA_API const char* mamba_version(void) { return "0.1.0"; }

}  // extern "C"
