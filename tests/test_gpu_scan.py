"""Selective scan: CUDA path (through the C ABI) vs the float64 oracle.

Element-by-element comparisons at sizes the oracle finishes in seconds (several
tiles, ragged tails, channel counts that are not a multiple of the 32-channel
warp group), and sampled chains at the full workload sizes in the launch
configuration the benchmark uses.
"""
import pytest
import torch

from oracle import oracle
from parity import BF16_TOL, FP32_TOL, max_rel_err, tol_for
from selective_state_space_55_b200 import inputs as I
from selective_state_space_55_b200 import ops

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def ref():
    return oracle.default()


def run_gpu(x, softplus=True, last=True, **kw):
    res = ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                                 delta_bias=x["delta_bias"], softplus=softplus,
                                 return_last_state=last, **kw)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    return res if last else (res, None)


def run_oracle(ref, x, softplus=True):
    cpu = {k: (None if v is None else v.cpu()) for k, v in x.items()}
    return ref.selective_scan(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"],
                              z=cpu["z"], delta_bias=cpu["delta_bias"], softplus=softplus)


def check(ref, x, tol, softplus=True, **kw):
    out, last = run_gpu(x, softplus=softplus, **kw)
    o_out, o_last = run_oracle(ref, x, softplus=softplus)
    e_out, e_last = max_rel_err(out, o_out), max_rel_err(last, o_last)
    assert e_out <= tol, f"out error {e_out:.3e} > {tol:.1e}"
    assert e_last <= tol, f"last_state error {e_last:.3e} > {tol:.1e}"
    return out, last


def layer_inputs(batch, dim, L, dtype=torch.bfloat16, bc=None, seed=0, N=16, recipe="layer"):
    cfg = I.SCAN_CONFIGS["mamba_1p4b_layer"].resized(batch=batch, dim=dim, seqlen=L, dstate=N,
                                                       io_dtype=dtype, bc_dtype=bc or dtype,
                                                       recipe=recipe)
    return I.make_scan_inputs(cfg, DEV, seed)


# ------------------------------------------------------------ configurations

def test_tiny_fp32_config(ref):
    cfg = I.SCAN_CONFIGS["tiny_fp32"]
    x = I.make_scan_inputs(cfg, DEV, seed=0)
    check(ref, x, FP32_TOL)


def test_layer_recipe_reduced_full_compare(ref):
    x = layer_inputs(2, 256, 2048)
    check(ref, x, BF16_TOL)


def test_layer_recipe_fp32_full_compare(ref):
    x = layer_inputs(2, 96, 1024, dtype=torch.float32)
    check(ref, x, FP32_TOL)


def sampled_check(ref, cfg, x, out, last, count, tol):
    for row in I.gather_chains(x, I.sample_chains(cfg.batch, cfg.dim, count, seed=3)):
        b, d = row["b"], row["d"]
        o_out, o_last = ref.selective_scan(row["u"], row["delta"], row["A"], row["B"], row["C"],
                                           D=row["D"], z=row["z"], delta_bias=row["delta_bias"],
                                           softplus=cfg.softplus)
        e = max_rel_err(out[b:b + 1, d:d + 1], o_out)
        assert e <= tol, f"chain ({b},{d}) out error {e:.3e}"
        if last is not None:
            e = max_rel_err(last[b:b + 1, d:d + 1], o_last)
            assert e <= tol, f"chain ({b},{d}) last_state error {e:.3e}"


@pytest.mark.parametrize("name", ["mamba_1p4b_layer", "mamba_2p8b_layer"])
def test_layer_config_full_size_sampled(ref, name):
    cfg = I.SCAN_CONFIGS[name]
    x = I.make_scan_inputs(cfg, DEV, seed=0)
    out, last = run_gpu(x, last=cfg.last_state)
    sampled_check(ref, cfg, x, out, last, 24, BF16_TOL)


def test_long_dna_config_full_size_sampled(ref):
    cfg = I.SCAN_CONFIGS["long_dna_1m"]
    x = I.make_scan_inputs(cfg, DEV, seed=0)
    out, last = run_gpu(x)
    plan = ops.scan_plan(cfg.batch, cfg.dim, cfg.dstate, cfg.seqlen,
                         sm_count=torch.cuda.get_device_properties(0).multi_processor_count)
    assert plan["nchunks"] > 1
    sampled_check(ref, cfg, x, out, last, 4, BF16_TOL)
    del x, out, last
    torch.cuda.empty_cache()


# ------------------------------------------------------------ segment carry

PAR = ops.MAMBA_FLAG_PARALLEL_CHUNKS                                 # three launches
PAR1 = ops.MAMBA_FLAG_PARALLEL_CHUNKS | ops.MAMBA_FLAG_PARALLEL_ONE_LAUNCH   # one launch, look-back
MODES = pytest.mark.parametrize("flags", [0, PAR, PAR1], ids=["chained", "parallel", "parallel1"])
PMODES = pytest.mark.parametrize("flags", [PAR, PAR1], ids=["parallel", "parallel1"])


@MODES
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("K", [2, 3, 8])
def test_segments_long_memory(ref, dtype, K, flags):
    """Tiny Delta makes the state carry across every segment boundary."""
    x = layer_inputs(1, 64, 4096, dtype=dtype, seed=K)
    x["delta_bias"] = torch.full_like(x["delta_bias"], -9.0)   # Delta ~ 1e-4
    out, last = check(ref, x, tol_for(dtype), num_chunks=K, flags=flags)
    ref_out, ref_last = run_gpu(x, num_chunks=1)
    assert max_rel_err(out, ref_out) <= tol_for(dtype)


@MODES
@pytest.mark.parametrize("L,K", [(100, 5), (1000, 3), (333, 4), (4096 + 40, 7)])
def test_segments_ragged(ref, L, K, flags):
    x = layer_inputs(2, 40, L, seed=L)
    check(ref, x, BF16_TOL, num_chunks=K, flags=flags)


def test_chained_segments_are_bitwise_single_pass():
    """Handing the state over through the workspace changes no arithmetic."""
    x = layer_inputs(3, 96, 2048, seed=30)
    a, la = run_gpu(x, num_chunks=1)
    for K in (2, 8, 128):
        b, lb = run_gpu(x, num_chunks=K)
        assert torch.equal(a, b) and torch.equal(la, lb)


@PMODES
def test_parallel_matches_single_pass_closely(ref, flags):
    x = layer_inputs(1, 32, 8192, dtype=torch.float32, seed=5)
    a, la = run_gpu(x, num_chunks=1)
    b, lb = run_gpu(x, num_chunks=16, flags=flags)
    assert max_rel_err(b, a) <= 1e-5 and max_rel_err(lb, la) <= 1e-5


@PMODES
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_parallel_correction_without_early_stop(ref, dtype, flags):
    """The parallel mode's correction walks a segment only while some
    exp(A_n S_t) is above fp32's range; with a state entry at A = 0 it never
    decays, so every segment is corrected to its end."""
    x = layer_inputs(2, 48, 3000, dtype=dtype, seed=43)
    A = x["A"].clone()
    A[:, 3] = 0.0
    x["A"] = A
    check(ref, x, tol_for(dtype), num_chunks=5, flags=flags)


@PMODES
def test_parallel_correction_with_negative_delta(ref, flags):
    """Softplus off with delta + bias of both signs: the running sum of Delta
    is not monotone, so the correction may not stop early."""
    x = layer_inputs(1, 64, 2048, dtype=torch.float32, seed=44)
    x["delta"] = (x["delta"] * 0.02).contiguous()
    x["delta_bias"] = torch.full_like(x["delta_bias"], 0.005)
    check(ref, x, FP32_TOL, softplus=False, num_chunks=6, flags=flags)


def test_many_groups_many_segments(ref):
    """More work items than resident warps, in both modes."""
    x = layer_inputs(4, 2048, 1024, seed=31)
    out, last = run_gpu(x, num_chunks=4)
    for flags in (0, PAR, PAR1):
        o2, l2 = run_gpu(x, num_chunks=4, flags=flags)
        assert max_rel_err(o2, out.double()) <= BF16_TOL
    sampled = I.SCAN_CONFIGS["mamba_1p4b_layer"].resized(batch=4, dim=2048, seqlen=1024)
    sampled_check(ref, sampled, x, out, last, 16, BF16_TOL)


def test_one_and_three_launch_parallel_modes_agree():
    """The look-back folds the earlier segments' states one after another, the
    three-launch form by a warp-shuffle scan: the same sums in another order."""
    x = layer_inputs(3, 96, 6000, seed=45)
    plan = ops.scan_plan(3, 96, 16, 6000, num_chunks=12, flags=PAR1,
                         sm_count=torch.cuda.get_device_properties(0).multi_processor_count)
    assert plan["mode"] == 2 and plan["launches"] == 1
    a, la = run_gpu(x, num_chunks=12, flags=PAR1)
    b, lb = run_gpu(x, num_chunks=12, flags=PAR)
    assert max_rel_err(a, b) <= BF16_TOL and max_rel_err(la, lb) <= 1e-5


def test_lookback_wait_reports_timeout():
    """Segments that never publish: every look-back gives up (bounded), the
    status word says MAMBA_ERR_TIMEOUT, and a normal call afterwards is fine."""
    x = layer_inputs(1, 64, 1024, seed=34)
    ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], num_chunks=4,
                           flags=PAR1 | ops.MAMBA_FLAG_TEST_WITHHOLD_HANDOFF)
    torch.cuda.synchronize()
    assert ops.device_status() == -6
    assert ops.device_status() == 0
    out, last = run_gpu(x, num_chunks=4, flags=PAR1)
    assert torch.isfinite(out.float()).all()


# ------------------------------------------------------------ edge cases

@pytest.mark.parametrize("L", [1, 2, 7, 8, 31, 33, 37, 40, 64, 65, 257])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_ragged_lengths(ref, L, dtype):
    x = layer_inputs(2, 48, L, dtype=dtype, seed=L)
    check(ref, x, tol_for(dtype))


@pytest.mark.parametrize("dim", [1, 16, 31, 33, 100])
def test_channel_counts(ref, dim):
    x = layer_inputs(3, dim, 96, seed=dim)
    check(ref, x, BF16_TOL)


@pytest.mark.parametrize("N", [1, 2, 4, 8, 13, 16])
def test_state_sizes(ref, N):
    x = layer_inputs(2, 64, 128, dtype=torch.float32, N=N, seed=N)
    check(ref, x, FP32_TOL)


@pytest.mark.parametrize("io,bc", [(torch.float32, torch.bfloat16), (torch.bfloat16, torch.float32)])
def test_mixed_dtypes(ref, io, bc):
    x = layer_inputs(2, 64, 256, dtype=io, bc=bc, seed=7)
    check(ref, x, tol_for(io))


@pytest.mark.parametrize("drop", ["z", "D", "delta_bias", "all"])
def test_optional_inputs(ref, drop):
    x = layer_inputs(2, 64, 256, dtype=torch.float32, seed=11)
    for k in (["z", "D", "delta_bias"] if drop == "all" else [drop]):
        x[k] = None
    check(ref, x, FP32_TOL)


def test_softplus_off(ref):
    x = layer_inputs(2, 64, 256, dtype=torch.float32, seed=12)
    x["delta"] = x["delta"].abs() * 0.1          # Delta = delta + bias must stay positive
    x["delta_bias"] = torch.rand_like(x["delta_bias"]) * 0.05
    check(ref, x, FP32_TOL, softplus=False)


def test_without_last_state(ref):
    x = layer_inputs(2, 64, 256, seed=13)
    out, _ = run_gpu(x, last=False)
    o_out, _ = run_oracle(ref, x)
    assert max_rel_err(out, o_out) <= BF16_TOL


def test_no_tma_path_is_bitwise_identical():
    x = layer_inputs(2, 96, 512, seed=14)
    a, la = run_gpu(x)
    b, lb = run_gpu(x, flags=ops.MAMBA_FLAG_NO_TMA)
    assert torch.equal(a, b) and torch.equal(la, lb)
    c, lc = run_gpu(x, num_chunks=3, flags=PAR)
    d, ld = run_gpu(x, num_chunks=3, flags=PAR | ops.MAMBA_FLAG_NO_TMA)
    assert torch.equal(c, d) and torch.equal(lc, ld)


def test_deterministic():
    x = layer_inputs(4, 128, 1024, seed=15)
    a, la = run_gpu(x)
    b, lb = run_gpu(x)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_empty_sequence_zeroes_last_state():
    x = layer_inputs(2, 64, 0)
    last = torch.full((2, 64, 16), 7.0, device=DEV)
    out = ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                                 delta_bias=x["delta_bias"], last_state=last)[0]
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.count_nonzero(last).item() == 0


def test_empty_batch():
    x = layer_inputs(0, 64, 32)
    out = ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"])
    assert out.numel() == 0


# ------------------------------------------------------------ the pages' limits on GPU

def test_gated_rnn_theorem1_on_gpu():
    """N = 1, A = -1, C = 1, B_t = g_t / Delta_t: h_t = (1 - g_t) h_{t-1} + g_t x_t."""
    g = torch.Generator().manual_seed(21)
    L, batch = 512, 3
    s = torch.randn(batch, 1, L, generator=g, dtype=torch.float64) * 2.0
    gate = torch.sigmoid(s)
    Delta = torch.nn.functional.softplus(s)
    xin = torch.randn(batch, 1, L, generator=g, dtype=torch.float64)
    want = torch.zeros_like(xin)
    h = torch.zeros(batch, 1, dtype=torch.float64)
    for t in range(L):
        h = (1 - gate[:, :, t]) * h + gate[:, :, t] * xin[:, :, t]
        want[:, :, t] = h
    f = lambda t: t.float().to(DEV).contiguous()  # noqa: E731
    out = ops.selective_scan_fwd(f(xin), f(s), -torch.ones(1, 1, device=DEV),
                                 f((gate / Delta).reshape(batch, 1, L)),
                                 torch.ones(batch, 1, L, device=DEV), softplus=True)
    assert max_rel_err(out, want) <= 1e-5


def test_large_delta_resets_state(ref):
    x = layer_inputs(2, 64, 128, dtype=torch.float32, seed=22)
    x["delta"] = torch.full_like(x["delta"], 1000.0)
    x["delta_bias"] = None
    out, last = check(ref, x, FP32_TOL, softplus=False)
    # h_t = Delta B_t u_t: last state depends only on the last token
    want = 1000.0 * x["B"][:, None, :, -1] * x["u"][:, :, -1][:, :, None]
    assert max_rel_err(last, want.double()) <= FP32_TOL


def test_small_delta_holds_state(ref):
    x = layer_inputs(2, 64, 200, dtype=torch.float32, seed=23)
    x["delta_bias"] = None
    x["delta"] = torch.full_like(x["delta"], -80.0)
    x["delta"][:, :, 0] = 40.0
    out, last = check(ref, x, FP32_TOL)
    h0 = 40.0 * x["B"][:, None, :, 0].double() * x["u"][:, :, 0][:, :, None].double()
    assert max_rel_err(last, h0) <= FP32_TOL


def test_zero_A_is_cumulative_sum(ref):
    x = layer_inputs(2, 64, 300, dtype=torch.float32, seed=24)
    x["A"] = torch.zeros_like(x["A"])
    check(ref, x, FP32_TOL)


def test_workspace_too_small_is_rejected():
    x = layer_inputs(1, 32, 4096)
    need = ops.scan_workspace_bytes(1, 32, 16, 4096, num_chunks=4)
    ws = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(ops.MambaError) as e:
        ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], num_chunks=4,
                               workspace=ws)
    assert e.value.status == -4


def test_workspace_reuse_across_calls():
    """The call clears its counters and flags itself: one workspace serves many calls."""
    x = layer_inputs(2, 64, 1024, seed=32)
    need = ops.scan_workspace_bytes(2, 64, 16, 1024, num_chunks=4)
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device=DEV)   # garbage to start with
    a = ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                               delta_bias=x["delta_bias"], num_chunks=4, workspace=ws)
    b = ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                               delta_bias=x["delta_bias"], num_chunks=4, workspace=ws)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    assert torch.equal(a, b)


def test_bounded_wait_reports_timeout():
    """A predecessor that never hands its state on: the waits give up, the
    status word says MAMBA_ERR_TIMEOUT, and the context stays usable."""
    x = layer_inputs(1, 64, 1024, seed=33)
    ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], num_chunks=4,
                           flags=ops.MAMBA_FLAG_TEST_WITHHOLD_HANDOFF)
    torch.cuda.synchronize()
    assert ops.device_status() == -6
    assert ops.device_status() == 0          # reading clears it
    out, last = run_gpu(x, num_chunks=4)     # a normal call afterwards is fine
    assert torch.isfinite(out.float()).all()
