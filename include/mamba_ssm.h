/*
 * mamba_ssm.h — C ABI of the B200 (sm_100a) selective-SSM library.
 *
 * Two operations, both from the Mamba selective state space model:
 *
 *   mamba_selective_scan_fwd      the selective scan over a whole sequence
 *   mamba_selective_state_update  one token of generation (recurrent mode)
 *
 * and, next to them, the block's short causal convolution (prefill and decode
 * update) that produces the scan's input.
 *
 * Definition (per batch b, channel d, state index n, time t):
 *
 *   Delta_t  = softplus(delta_t + delta_bias_d)      (or without softplus)
 *   Abar     = exp(Delta_t * A_d,n)
 *   h_t,n    = Abar * h_{t-1},n + Delta_t * B_t,n * u_t        h_{-1} = 0
 *   y_t      = sum_n C_t,n * h_t,n + D_d * u_t
 *   out_t    = y_t * silu(z_t)                                   (z optional)
 *
 * Options: MAMBA_FLAG_ZOH replaces the Euler input term Delta_t B_t,n u_t by
 * the zero-order-hold one, expm1(Delta_t A_d,n) / A_d,n * B_t,n * u_t
 * (Delta_t B_t,n u_t where A_d,n = 0); mamba_selective_scan_fwd_with_state
 * starts from a given h_{-1} instead of zero.
 *
 * Sources: "超越注意力：探索Mamba与状态空间模型" (ai-lab.club), section
 * 状态空间模型基础 (zero-order-hold Abar = exp(Delta A), recurrence and
 * readout, and the zero-order-hold Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B
 * of MAMBA_FLAG_ZOH) and section 选择性状态空间模型 (Delta = softplus(W x + b),
 * B and C per token); its section 代码实现概览 uses the Euler input term
 * Bbar = Delta * B, the default here.  "Mamba 与状态空间模型"
 * (world.lapla.si), section 由词元决定 (exp(Delta A) decides how much old state
 * is kept) and section 在芯片上扫过去 (the scan never writes the full state to
 * HBM).  The silu(z) gate is the Mamba block's output gate (not printed on the
 * pages).  The update is the same step applied once to a stored state
 * ("Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
 * (mentras.net), table 复杂度对比: constant work per generated token).
 *
 * Conventions shared by every entry point
 *  - Pointers named in the signatures are DEVICE pointers owned by the caller;
 *    the dims struct is a HOST pointer.  The library keeps no per-call state
 *    and performs no device allocation.  Work is enqueued on `stream`
 *    (asynchronous); pass 0 for the legacy default stream.
 *  - All tensors are dense, row-major, contiguous, without padding.
 *  - Floating-point arithmetic is fp32; the state is fp32.  u/delta/z/out
 *    (x/dt/z/out) and B/C may each be fp32 or bf16 (see mamba_dtype_t).
 *    A, D and the delta/dt bias are fp32.
 *  - Return value: MAMBA_OK, or a negative mamba_status_t.  Argument errors
 *    are detected before anything is launched.  MAMBA_ERR_CUDA reports a
 *    launch failure (cudaGetLastError after the launch).  Faults that happen
 *    later on the device surface at the next synchronising CUDA call;
 *    mamba_device_status() reports the library's own device-side checks.
 *  - Outputs must not alias inputs (except the in-place state of the update).
 */
#ifndef MAMBA_SSM_H
#define MAMBA_SSM_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define MAMBA_API __declspec(dllexport)
#else
#define MAMBA_API __attribute__((visibility("default")))
#endif

typedef enum {
    MAMBA_OK = 0,
    MAMBA_ERR_INVALID_ARG = -1,   /* null required pointer, negative size, ... */
    MAMBA_ERR_UNSUPPORTED = -2,   /* dtype code, or dstate outside 1..16 */
    MAMBA_ERR_ALIGN = -3,         /* a pointer is not aligned to its element size */
    MAMBA_ERR_WORKSPACE = -4,     /* workspace missing or smaller than required */
    MAMBA_ERR_CUDA = -5,          /* a CUDA runtime call failed */
    MAMBA_ERR_TIMEOUT = -6,       /* a bounded device-side wait gave up */
    MAMBA_ERR_TOO_LARGE = -7      /* needs more scratch than the built-in array holds */
} mamba_status_t;

typedef enum {
    MAMBA_F32 = 0,
    MAMBA_BF16 = 1
} mamba_dtype_t;

/* Flags (mamba_dims_t.flags). */
#define MAMBA_FLAG_NO_TMA 0x1          /* plain loads instead of TMA (scan tiles; the
                                          * update's bulk streaming path) */
#define MAMBA_FLAG_PARALLEL_CHUNKS 0x2 /* with num_chunks >= 1: parallel mode (segments at
                                          * once, carry scan, correction) */
/* Test only: in mode 0, segments never hand their state on, so every wait for
 * a predecessor runs out (after ~0.3 s) and the call reports MAMBA_ERR_TIMEOUT
 * through mamba_device_status().  Outputs are then undefined. */
#define MAMBA_FLAG_TEST_WITHHOLD_HANDOFF 0x4
/* Scan and update: zero-order-hold input term expm1(Delta A) / A * B * u
 * instead of the Euler Delta * B * u (Abar = exp(Delta A) either way).  The scan
 * then runs a kernel instance with 1/A held in registers (fewer resident
 * warps); results follow the same tolerance as the Euler path. */
#define MAMBA_FLAG_ZOH 0x8
/* Update only: launch the streaming kernel as a programmatic dependent launch,
 * so that it may start while the previous kernel on the stream finishes.  It
 * reads its own state before waiting for that kernel, and x, dt, z, B, C after
 * it completes.  Set it only when the previous kernel on the stream does not
 * write this call's state, as when consecutive calls update the states of
 * different layers; then results are identical with and without the flag.
 * Paths other than the streaming one ignore it. */
#define MAMBA_FLAG_PDL 0x10
/* Scan forward (mamba_selective_scan_fwd, _with_state, _noalloc and the
 * host-buffer call) and backward: u, delta, z and out (dout and the
 * gradients du, ddelta, dz) are (batch, seqlen, dim), dim fastest,
 * the activation layout of the sample module in "超越注意力：探索Mamba与状态空间
 * 模型", section 代码实现概览; B and C stay (batch, dstate, seqlen) and the
 * states (batch, dim, dstate).  Tiles of (steps x 32 channels) are staged by
 * TMA (dim * element size a multiple of 16 bytes, 16-byte aligned pointers;
 * otherwise plain loads) and transposed on chip; outputs are stored one step
 * at a time.  Such calls always run in mode 0: MAMBA_FLAG_PARALLEL_CHUNKS with
 * it returns MAMBA_ERR_UNSUPPORTED.  The backward stages (8 steps x 32
 * channels) tiles by cp.async and stores its gradients one step at a time. */
#define MAMBA_FLAG_LAYOUT_BLD 0x20
/* Scan forward: keep one lane per channel where the plan would give each
 * channel two lanes (plan.lanes_per_channel; see mamba_scan_plan_t).  For
 * tests and measurements; results agree to rounding either way. */
#define MAMBA_FLAG_ONE_LANE_PER_CHANNEL 0x40
/* Scan, parallel mode: run it as one launch in which each segment looks back
 * at the earlier segments of its channel group and corrects its own outputs
 * (plan.mode 2), instead of three launches (segments, a warp-shuffle scan of
 * the segments' carries, a correction pass; plan.mode 1).  Results agree to
 * rounding.  Not the default: the one-launch form measured slower (the
 * correction shares the scan kernel's registers). */
#define MAMBA_FLAG_PARALLEL_ONE_LAUNCH 0x80

#define MAMBA_MAX_DSTATE 16

/*
 * Sizes and options of one call.
 *   batch, dim, dstate   B, D (channels) and N (state size, 1..16)
 *   seqlen               L for the scan; ignored by the update
 *   io_dtype             dtype of u, delta, z, out (update: x, dt, z, out)
 *   bc_dtype             dtype of B and C
 *   dt_softplus          update only: apply softplus to dt + dt_bias (0/1)
 *   num_chunks           scan only: 0 = automatic; k >= 1 forces the sequence
 *                        to be split into k segments (k = 1: one segment)
 *   flags                MAMBA_FLAG_*
 *   workspace            scan only: device scratch of at least
 *                        mamba_selective_scan_workspace_bytes() bytes, 256-byte
 *                        aligned, owned by the caller.  The call zeroes a few KB
 *                        at its start (counters, flags) on `stream`; concurrent
 *                        calls need separate workspaces.
 */
typedef struct {
    int64_t batch;
    int64_t dim;
    int64_t dstate;
    int64_t seqlen;
    int32_t io_dtype;
    int32_t bc_dtype;
    int32_t dt_softplus;
    int32_t num_chunks;
    int32_t flags;
    int32_t reserved;
    void *workspace;
    size_t workspace_bytes;
} mamba_dims_t;

/*
 * How a scan call will run (host-side planning; no CUDA call is made).
 * The channels form groups of 32 (one warp each, one channel per lane), or of
 * 16 with two lanes per channel when 32-channel groups would leave resident
 * warps idle in mode 0; the sequence is cut into
 * nchunks segments of chunk_len steps (the last may be shorter).  A persistent
 * grid of warps pulls (segment, group) work items from a counter.
 *   mode 0 (chained): one launch.  Segment k of a group starts from the state
 *     segment k-1 left in the workspace; no work is repeated.  Used when there
 *     are enough groups to occupy the GPU; nchunks only balances the load.
 *   mode 1 (parallel): three launches, for few channels and long sequences.
 *     1. Every segment runs at once from a zero start (segment 0 from the
 *        start state), writes its outputs and keeps its end state and its
 *        sum of Delta (units_pass_a items).
 *     2. One warp per chain scans the segments' (exp(A sum Delta), end state)
 *        pairs with warp shuffles (the associative combine of the parallel
 *        scan): each segment's true start state, and last_state.
 *     3. Each later segment adds its start state's contribution,
 *        C_t . (exp(A S_t) h_in) with S_t the sum of Delta since the segment
 *        began, to its outputs (units_pass_b items, one per chain and
 *        segment), stopping where exp(A S_t) has underflowed in fp32 for
 *        every state entry (when Delta >= 0 throughout, i.e. softplus on).
 *     Nothing is computed twice; the correction costs as much per step as
 *     the scan but covers only the steps over which the start state matters.
 *   mode 2 (parallel, with MAMBA_FLAG_PARALLEL_ONE_LAUNCH): the same work in one launch.
 *     After step 1 each segment publishes its end state and sum of Delta,
 *     waits (bounded) for the earlier segments of its channel group to have
 *     published theirs (a decoupled look-back: segments are taken in order,
 *     so the earlier ones always run), folds them into its own start state,
 *     and corrects its own outputs (units_pass_b corrections, inside the
 *     launch).
 */
typedef struct {
    int32_t nchunks;           /* segments per sequence */
    int32_t tile_len;          /* time steps staged per pipeline stage */
    int64_t chunk_len;         /* time steps per segment (multiple of tile_len) */
    int64_t groups;            /* batch * ceil(dim / (32 / lanes_per_channel)) */
    int64_t units_pass_a;      /* work items of the first launch (group x segment) */
    int64_t units_pass_b;      /* correction items, chain x later segment (0 in mode 0) */
    int32_t warps_per_cta;
    int32_t launches;          /* kernel launches per call (plus one memset): 1 or 3 */
    int32_t tma_capable;       /* strides allow TMA staging */
    int32_t mode;              /* 0 chained, 1 parallel (three launches), 2 parallel (one launch) */
    int32_t channels_per_lane; /* 1 or 2: a group is 32 x this many channels */
    int32_t lanes_per_channel; /* 1, or 2 when a group is 16 channels whose 16 state
                                * entries are split over two lanes (mode 0 with fewer
                                * 32-channel groups than resident warps, Euler input
                                * term, (batch, dim, seqlen) layout) */
    int64_t max_warps;         /* warps the persistent grid uses at most */
    size_t workspace_bytes;
} mamba_scan_plan_t;

/*
 * Plan a scan for `dims` on a GPU with `sm_count` SMs.  Pure host function.
 * Returns MAMBA_ERR_INVALID_ARG / MAMBA_ERR_UNSUPPORTED for bad dims.
 */
MAMBA_API mamba_status_t mamba_selective_scan_plan(const mamba_dims_t *dims, int sm_count,
                                                   mamba_scan_plan_t *plan);

/*
 * Scratch bytes mamba_selective_scan_fwd needs for `dims` on the current
 * device: a few KB of counters and flags plus the segment carry (64 bytes per
 * chain in mode 0, 68 bytes per chain and segment in mode 1).  0 for empty
 * problems.  Returns (size_t)-1 on bad dims or when the current device cannot
 * be queried.
 */
MAMBA_API size_t mamba_selective_scan_workspace_bytes(const mamba_dims_t *dims);

/*
 * Selective scan forward.
 *   u, delta, z, out   (batch, dim, seqlen), io_dtype; z may be NULL (no gate);
 *                      (batch, seqlen, dim) with MAMBA_FLAG_LAYOUT_BLD
 *   A                  (dim, dstate) fp32
 *   B, C               (batch, dstate, seqlen), bc_dtype, shared by all channels
 *   D, delta_bias      (dim,) fp32; may be NULL (treated as 0)
 *   softplus           nonzero: Delta = softplus(delta + delta_bias)
 *   last_state         (batch, dim, dstate) fp32 = h at t = seqlen-1; may be NULL
 *   dims->workspace    required (see mamba_selective_scan_workspace_bytes)
 * seqlen == 0 writes no output; last_state (if given) is set to zero.
 * Returns MAMBA_ERR_WORKSPACE if the workspace is missing or too small.
 * Sources: the recurrence h_t = Abar h_{t-1} + Bbar x_t, y_t = C h_t with
 * Abar = exp(Delta A), "超越注意力：探索Mamba与状态空间模型", section
 * 状态空间模型基础; Delta = softplus(. + b) and B, C per token, the same page,
 * section 选择性状态空间模型, and Bbar x = Delta B u as in its section
 * 代码实现概览; the scan that keeps the state on chip and writes only the
 * outputs, "Mamba 与状态空间模型", section 在芯片上扫过去.
 */
MAMBA_API mamba_status_t mamba_selective_scan_fwd(const void *u, const void *delta, const float *A,
                                                  const void *B, const void *C, const float *D,
                                                  const void *z, const float *delta_bias,
                                                  int softplus, void *out, float *last_state,
                                                  const mamba_dims_t *dims, cudaStream_t stream);

/*
 * Selective scan forward from a given start state.
 *
 * Same as mamba_selective_scan_fwd, except that the recurrence starts from
 *   initial_state      (batch, dim, dstate) fp32 device buffer = h_{-1}, or NULL
 *                      for the zero state (then identical to
 *                      mamba_selective_scan_fwd).
 * A sequence can thus be scanned in pieces: the last_state of one call is the
 * initial_state of the next, and the outputs equal those of one call over the
 * whole sequence up to rounding.  initial_state may be the same buffer as
 * last_state (it is read before last_state is written); a partial overlap of
 * the two returns MAMBA_ERR_INVALID_ARG.  With seqlen == 0, last_state (if
 * given) receives a copy of initial_state (zero if NULL).
 * Source: the recurrence of "超越注意力：探索Mamba与状态空间模型", section
 * 状态空间模型基础, from an arbitrary h_{t-1}; "Mamba 与状态空间模型", section
 * 固定大小的状态 (the fixed-size state carries everything the model keeps).
 */
MAMBA_API mamba_status_t mamba_selective_scan_fwd_with_state(
    const void *u, const void *delta, const float *A, const void *B, const void *C,
    const float *D, const void *z, const float *delta_bias, int softplus,
    const float *initial_state, void *out, float *last_state, const mamba_dims_t *dims,
    cudaStream_t stream);

/*
 * Selective scan forward over HOST buffers, with the copies pipelined.
 *
 * For callers whose activations live in host memory: the batch is cut into
 * chunks of `rows` batch rows; while chunk c is scanned, chunk c+1 is being
 * copied in and chunk c-1 copied out, on two internal streams, so that the
 * host-to-device and device-to-host transfers (the bound for this use) run at
 * the same time and hide the scan.  Each chunk is one scan over its rows,
 * identical in definition to mamba_selective_scan_fwd_with_state.
 *   u, delta, z, B, C, A, D, delta_bias, initial_state     HOST pointers (read)
 *   out, last_state                                        HOST pointers (written)
 *     Same shapes, dtypes, optional (NULL) arguments and meaning as in
 *     mamba_selective_scan_fwd_with_state.  Page-locked (pinned) host memory
 *     is needed for the copies to overlap; pageable memory gives the same
 *     results, without the overlap.
 *   rows               batch rows per chunk; 0 = automatic (about 8 chunks)
 *   dims->workspace    DEVICE scratch of at least
 *                      mamba_selective_scan_host_workspace_bytes(dims, rows)
 *                      bytes, 256-byte aligned: three chunk stages (their
 *                      inputs, outputs and scan scratch) and A, D, delta_bias.
 *   stream             the scans run on it; the call is ordered after earlier
 *                      work on `stream`, and later work on `stream` is ordered
 *                      after the last copy back to the host.  The call returns
 *                      once everything is enqueued; host results are complete
 *                      when `stream` has been synchronised.
 * The two copy streams and their events are created on first use per device
 * and kept; enqueueing is serialised by a lock, so calls from several host
 * threads are safe but do not overlap each other's copies.
 * Returns MAMBA_ERR_INVALID_ARG for rows < 0 or missing required pointers,
 * MAMBA_ERR_WORKSPACE if the workspace is missing or too small.
 * The paper has no counterpart; it is the host side of the same scan.
 */
MAMBA_API size_t mamba_selective_scan_host_workspace_bytes(const mamba_dims_t *dims, int64_t rows);

MAMBA_API mamba_status_t mamba_selective_scan_fwd_host(
    const void *u, const void *delta, const float *A, const void *B, const void *C,
    const float *D, const void *z, const float *delta_bias, int softplus,
    const float *initial_state, void *out, float *last_state, int64_t rows,
    const mamba_dims_t *dims, cudaStream_t stream);

/*
 * Selective scan forward that allocates nothing and takes no workspace.
 *
 * The paper has no counterpart to this entry point; it is a deployment aid.
 * Some callers cannot allocate device memory: a host program whose device
 * memory is owned by another allocator (a framework's caching allocator, a
 * fixed arena) that forbids outside cudaMalloc calls, or latency-critical
 * code that cannot pay for cudaMalloc/cudaFree and the device
 * synchronisation they may imply.  This variant runs the same kernel as
 * mamba_selective_scan_fwd with its scratch in a static device array of
 * MAMBA_NOALLOC_SCRATCH_BYTES (8 MiB) that every GPU which loads the library
 * holds until the process exits.  The caller still provides every input and
 * output buffer; dims->workspace and dims->workspace_bytes are ignored.
 *
 *  - Arguments, layouts and results are those of mamba_selective_scan_fwd.
 *  - Problems whose plan needs more than MAMBA_NOALLOC_SCRATCH_BYTES of
 *    scratch are refused with MAMBA_ERR_TOO_LARGE before anything is
 *    launched.  8 MiB covers, for example, chained segments of up to
 *    131,000 (batch x channel) chains, which includes the Mamba-2.8B layer
 *    shape (81,920 chains).
 *  - The first call on each device looks up the array's device address with
 *    cudaGetSymbolAddress, with that device current, and keeps it for the
 *    life of the process.  Make that first call before any stream capture.
 *    The kept address does not survive cudaDeviceReset: after resetting a
 *    device, do not call this entry point on it again in the same process.
 *  - Every call, on every stream, shares the one array per device.  Each call
 *    clears the part that must start at zero, but calls whose executions
 *    overlap on the GPU race on the array: run them in one stream or otherwise
 *    one after another.
 *  - Never calls cudaMalloc, cudaFree or any allocating library routine.
 */
#define MAMBA_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

MAMBA_API mamba_status_t mamba_selective_scan_fwd_noalloc(
    const void *u, const void *delta, const float *A, const void *B, const void *C,
    const float *D, const void *z, const float *delta_bias, int softplus, void *out,
    float *last_state, const mamba_dims_t *dims, cudaStream_t stream);

/*
 * Single-token state update (generation).  The state is read and written in
 * place.
 *   state              (batch, dim, dstate) fp32, updated in place
 *   x, dt, z, out      (batch, dim), io_dtype; z may be NULL
 *   A                  (dim, dstate) fp32
 *   B, C               (batch, dstate), bc_dtype
 *   D, dt_bias         (dim,) fp32; may be NULL
 *   dims->dt_softplus  nonzero: Delta = softplus(dt + dt_bias)
 *   dims->flags        MAMBA_FLAG_ZOH: zero-order-hold input term
 * dims->seqlen, num_chunks and workspace are ignored.
 * Paths: for dstate == 16, dim % 8 == 0 and 16-byte aligned buffers the state
 * streams through shared memory by bulk TMA (MAMBA_FLAG_NO_TMA turns that
 * off); otherwise plain vectorised loads (dstate == 16) or a scalar path.
 * Sources: one step of the recurrence of "超越注意力：探索Mamba与状态空间模型",
 * sections 状态空间模型基础 and 选择性状态空间模型, applied to a stored state;
 * "Mamba: Linear-Time Sequence Modeling with Selective State Spaces", table
 * 复杂度对比 (constant time and memory per generated token); "Mamba 与状态空间模型",
 * section 固定大小的状态 (the fixed-size state is all that generation keeps).
 */
MAMBA_API mamba_status_t mamba_selective_state_update(float *state, const void *x, const void *dt,
                                                      const float *A, const void *B, const void *C,
                                                      const float *D, const void *z,
                                                      const float *dt_bias, void *out,
                                                      const mamba_dims_t *dims,
                                                      cudaStream_t stream);

/*
 * Backward pass of the selective scan (training).
 *
 * Gradients of a scalar loss, given dout = dLoss/dout (and optionally
 * dlast_state = dLoss/dlast_state), with respect to every input of
 * mamba_selective_scan_fwd_with_state, with the Euler input term or, with
 * MAMBA_FLAG_ZOH in dims->flags, the zero-order-hold one (with
 * MAMBA_FLAG_LAYOUT_BLD, u, delta, z, dout and du, ddelta, dz are
 * (batch, seqlen, dim)).  As in the pages'
 * description of the hardware-aware scan ("Mamba 与状态空间模型", section
 * 在芯片上扫过去), the per-step states are not stored by the forward: a
 * checkpoint pass keeps the state every 8 steps in the workspace, and the
 * backward recomputes the states in between from it.  With
 * lambda_t = dLoss/dh_t the adjoint runs backwards in time:
 *   lambda_t = C_t dy_t + Abar_t+1 lambda_t+1,   dy = dout * silu(z)
 *   dC_t,n = dy_t h_t,n;  dB_t,n = lambda_t,n Delta_t u_t
 *   dDelta_t = sum_n lambda_t,n (B_t,n u_t + A_n Abar_t,n h_t-1,n)  (then * softplus')
 *   dA_n = sum_t lambda_t,n Delta_t Abar_t,n h_t-1,n;  du_t = D dy_t + Delta_t sum_n lambda_t,n B_t,n
 * With the zero-order hold the input gain g = expm1(Delta A) / A replaces Delta
 * in the input term ("超越注意力：探索Mamba与状态空间模型", section 状态空间模型基础):
 * dB = lambda g u, du = D dy + sum_n lambda g B, dDelta gains Abar B u in place
 * of B u (dg/dDelta = Abar) and dA gains lambda dg/dA B u with
 * dg/dA = (Delta Abar - g) / A (its series near Delta A = 0, limit Delta^2 / 2).
 * Inputs (device): the forward's inputs (u, delta, A, B, C, D, z, delta_bias,
 *   softplus, initial_state: same shapes, dtypes and NULL rules), dout
 *   (batch, dim, seqlen) io_dtype, dlast_state (batch, dim, dstate) fp32 or NULL.
 * Outputs (device, overwritten): du, ddelta, dz (batch, dim, seqlen) io_dtype;
 *   dA (dim, dstate), dB and dC (batch, dstate, seqlen), dD and ddelta_bias
 *   (dim,), dinitial_state (batch, dim, dstate), all fp32.  dz, dD,
 *   ddelta_bias and dinitial_state may be NULL (not computed); dz needs z.
 *   dA, dB, dC, dD and ddelta_bias are sums over many channels and time
 *   steps, accumulated with atomic adds: their rounding order (not their
 *   value) varies from run to run.
 * dims->workspace: at least mamba_selective_scan_bwd_workspace_bytes(dims)
 *   bytes, 256-byte aligned (64 bytes per chain and 8 steps for the
 *   checkpoints, plus the segment handoffs).
 * Segments of a sequence are processed one after another (chained), so
 * sequences much longer than the batch x channel count can keep busy run with
 * little parallelism.
 */
MAMBA_API size_t mamba_selective_scan_bwd_workspace_bytes(const mamba_dims_t *dims);

MAMBA_API mamba_status_t mamba_selective_scan_bwd(
    const void *u, const void *delta, const float *A, const void *B, const void *C,
    const float *D, const void *z, const float *delta_bias, int softplus,
    const float *initial_state, const void *dout, const float *dlast_state, void *du,
    void *ddelta, float *dA, float *dB, float *dC, float *dD, void *dz, float *ddelta_bias,
    float *dinitial_state, const mamba_dims_t *dims, cudaStream_t stream);

/*
 * Short causal convolution of the Mamba block.
 *
 * Besides its 16 state numbers, each channel keeps a short convolution over
 * its most recent inputs ("Mamba 与状态空间模型", section 固定大小的状态: 4 of
 * them in Mamba-2.8B).  Per channel d, with W = width taps:
 *
 *   out_t = act(bias_d + sum_{k<W} weight_d,k * x_{t-W+1+k}),   act = silu or identity
 *
 * where x at negative times comes from a conv state holding the W most recent
 * inputs, oldest first (zero when no state is given).  In the block the conv
 * output feeds the projections that produce Delta, B and C, so it runs before
 * the scan (prefill) or the state update (decode), not inside them.
 *
 * mamba_causal_conv1d_fwd (prefill over a sequence)
 *   x, out              (batch, dim, seqlen), io_dtype; out must not alias x
 *   weight              (dim, width) fp32;  bias (dim,) fp32 or NULL
 *   initial_conv_state  (batch, dim, width), io_dtype, or NULL (zeros)
 *   final_conv_state    (batch, dim, width), io_dtype, or NULL: the last
 *                       width inputs of (initial state ++ x); may be the
 *                       initial_conv_state buffer itself (partial overlap:
 *                       MAMBA_ERR_INVALID_ARG)
 *   silu                nonzero: act = silu
 * mamba_causal_conv1d_update (one token of generation)
 *   conv_state          (batch, dim, width), io_dtype, updated in place: shifted
 *                       by one with x appended, then used for the sum
 *   x, out              (batch, dim), io_dtype
 * dims: batch, dim, seqlen (prefill) and io_dtype are read; dstate, bc_dtype
 * and the workspace are ignored.  For the update, dims->flags may hold
 * MAMBA_FLAG_PDL: with width 4 and conv_state, x and out aligned to their
 * vectors, the update is then launched as a programmatic dependent launch that
 * may start while the previous kernel on the stream finishes; it reads its own
 * conv_state first and waits for that kernel before it reads x or writes
 * anything.  Set it only when the previous kernel neither reads nor writes this
 * call's conv_state (consecutive layers of a decode step); results are then
 * identical with and without it.  width must be 1..MAMBA_MAX_CONV_WIDTH
 * (MAMBA_ERR_UNSUPPORTED otherwise).  Both calls are asynchronous on `stream`
 * and allocate nothing.
 */
#define MAMBA_MAX_CONV_WIDTH 4

MAMBA_API mamba_status_t mamba_causal_conv1d_fwd(const void *x, const float *weight,
                                                 const float *bias,
                                                 const void *initial_conv_state, int width,
                                                 int silu, void *out, void *final_conv_state,
                                                 const mamba_dims_t *dims, cudaStream_t stream);

MAMBA_API mamba_status_t mamba_causal_conv1d_update(void *conv_state, const void *x,
                                                    const float *weight, const float *bias,
                                                    int width, int silu, void *out,
                                                    const mamba_dims_t *dims,
                                                    cudaStream_t stream);

/*
 * Mamba-2 layer: the selective state space with a scalar A per head
 * ("Mamba 与状态空间模型", section "Mamba-2：两种算法": A is one number times
 * the identity, the layer applies one lower-triangular matrix whose entry
 * (i, j) is C_i . B_j times the decay between the steps, and a chunked
 * algorithm does dense products inside chunks and passes only the state
 * between them).  For each batch b and head h, with group g = h / (nheads /
 * ngroups) and the state S a (headdim x dstate) matrix:
 *
 *   Delta_t = softplus(dt_t,h + dt_bias_h)     (dt + dt_bias if dt_softplus == 0)
 *   S_t     = exp(Delta_t A_h) S_{t-1} + Delta_t x_t,h B_t,g^T,   S_{-1} = initial_state or 0
 *   out_t,h = (S_t C_t,g + D_h x_t,h) * silu(z_t,h)            (no gate when z == NULL)
 *
 * Arguments (all device pointers, caller-owned, contiguous row-major):
 *   x, z, out      (batch, seqlen, nheads, headdim) bf16; z may be NULL;
 *                  out must not alias an input
 *   dt             (batch, seqlen, nheads) bf16
 *   A              (nheads,) fp32, expected <= 0
 *   B, C           (batch, seqlen, ngroups, dstate) bf16
 *   D, dt_bias     (nheads,) fp32 or NULL
 *   initial_state  (batch, nheads, headdim, dstate) fp32 or NULL (zeros)
 *   final_state    (batch, nheads, headdim, dstate) fp32 or NULL: S at the
 *                  last step (initial_state, or zeros, when seqlen == 0)
 * Delta must not be negative: with dt_softplus == 0 the caller guarantees
 * dt + dt_bias >= 0 (a negative Delta gives undefined output).
 *
 * Supported shape: headdim == 64 and dstate == 128 (the published Mamba-2
 * models' head and state sizes), io_dtype MAMBA_BF16, ngroups dividing
 * nheads; anything else returns MAMBA_ERR_UNSUPPORTED (or
 * MAMBA_ERR_INVALID_ARG for negative sizes, missing required pointers or
 * ngroups not dividing nheads) before anything is launched.  x, z, out, B and
 * C must be 16-byte aligned, the fp32 arrays 4-byte aligned and dt 2-byte
 * aligned (MAMBA_ERR_ALIGN).  Products run on the tensor cores with bf16
 * operands and fp32 accumulation.  The operands the kernel computes (the
 * masked intra-chunk matrix, the weighted input and the copy of the entering
 * state) are each carried as a bf16 hi/lo pair (about 16 significant bits),
 * so the carried state stays fp32-accurate and the only bf16-level rounding
 * of the output is its own.
 * Asynchronous on `stream`; allocates nothing; a device-side wait that gives
 * up is reported by mamba_device_status() as MAMBA_ERR_TIMEOUT.
 */
typedef struct {
    int64_t batch, seqlen, nheads, headdim, ngroups, dstate;
    mamba_dtype_t io_dtype;   /* x, dt, z, out, B, C */
    int32_t dt_softplus;      /* nonzero: Delta = softplus(dt + dt_bias) */
} mamba_ssd_dims_t;

MAMBA_API mamba_status_t mamba_ssd_chunk_scan_fwd(const void *x, const void *dt, const float *A,
                                                  const void *B, const void *C, const float *D,
                                                  const void *z, const float *dt_bias,
                                                  const float *initial_state, void *out,
                                                  float *final_state,
                                                  const mamba_ssd_dims_t *dims,
                                                  cudaStream_t stream);

/*
 * Read and clear the library's device-side status word on the current device
 * (synchronises the device).  Returns MAMBA_OK, or the first device-side
 * error recorded since the last call (e.g. MAMBA_ERR_TIMEOUT).
 */
MAMBA_API mamba_status_t mamba_device_status(void);

/* Static, human-readable name of a status code. */
MAMBA_API const char *mamba_status_string(mamba_status_t status);

/* Library version as "major.minor.patch". */
MAMBA_API const char *mamba_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MAMBA_SSM_H */
