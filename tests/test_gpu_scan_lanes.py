"""The scan's two kernels on the same inputs: one lane per channel, and two
lanes per channel (each lane 8 of the 16 state entries, the softplus and the
readout halves swapped between the lanes).  The planner gives small chained
problems two lanes, so the other scan tests run that kernel on their small
shapes and the one-lane kernel on the full-size ones; here both run on each
small case (MAMBA_FLAG_ONE_LANE_PER_CHANNEL selects the one-lane kernel) and
both are held to the float64 oracle."""
import pytest
import torch

from oracle import oracle
from parity import max_rel_err, tol_for
from selective_state_space_55_b200 import inputs as I
from selective_state_space_55_b200 import ops

pytestmark = pytest.mark.gpu

DEV = "cuda"
ONE = ops.MAMBA_FLAG_ONE_LANE_PER_CHANNEL


@pytest.fixture(scope="module")
def ref():
    return oracle.default()


def inputs(batch, dim, L, dtype=torch.bfloat16, bc=None, seed=0, N=16):
    cfg = I.SCAN_CONFIGS["mamba_1p4b_layer"].resized(batch=batch, dim=dim, seqlen=L, dstate=N,
                                                       io_dtype=dtype, bc_dtype=bc or dtype,
                                                       recipe="layer")
    return I.make_scan_inputs(cfg, DEV, seed)


def lanes_of(x, flags=0, num_chunks=0):
    b, d, L = x["u"].shape
    return ops.scan_plan(b, d, x["A"].shape[1], L, x["u"].dtype, x["B"].dtype,
                         num_chunks=num_chunks, flags=flags,
                         sm_count=torch.cuda.get_device_properties(0).multi_processor_count
                         )["lanes_per_channel"]


def run(x, softplus=True, flags=0, **kw):
    out, last = ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"],
                                       z=x["z"], delta_bias=x["delta_bias"], softplus=softplus,
                                       return_last_state=True, flags=flags, **kw)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    return out, last


def both(ref, x, softplus=True, **kw):
    """Run both kernels, check each against the oracle; returns the outputs."""
    assert lanes_of(x, num_chunks=kw.get("num_chunks", 0)) == 2
    assert lanes_of(x, ONE, kw.get("num_chunks", 0)) == 1
    c = {k: (None if v is None else v.cpu()) for k, v in x.items()}
    o_out, o_last = ref.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], D=c["D"],
                                       z=c["z"], delta_bias=c["delta_bias"], softplus=softplus)
    tol = tol_for(x["u"].dtype)
    res = {}
    for name, flags in (("two", 0), ("one", ONE)):
        out, last = run(x, softplus=softplus, flags=flags, **kw)
        e_out, e_last = max_rel_err(out, o_out), max_rel_err(last, o_last)
        assert e_out <= tol, f"{name} lanes: out error {e_out:.3e} > {tol:.1e}"
        assert e_last <= tol, f"{name} lanes: last_state error {e_last:.3e} > {tol:.1e}"
        res[name] = (out, last)
    return res


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("L", [1, 7, 8, 9, 33, 100, 257, 1000])
def test_ragged_lengths(ref, dtype, L):
    both(ref, inputs(2, 48, L, dtype=dtype, seed=L))


@pytest.mark.parametrize("dim", [1, 15, 16, 17, 31, 100])
def test_channel_counts(ref, dim):
    """Groups of 16 with a partial last group, and lone channels."""
    both(ref, inputs(3, dim, 300, seed=dim))


@pytest.mark.parametrize("N", [1, 5, 8, 9, 16])
def test_state_sizes(ref, N):
    """N <= 8 leaves the second lane of each channel with padding only."""
    both(ref, inputs(2, 64, 512, N=N, seed=N))


@pytest.mark.parametrize("io,bc", [(torch.float32, torch.bfloat16), (torch.bfloat16, torch.float32)])
def test_mixed_dtypes(ref, io, bc):
    both(ref, inputs(2, 64, 400, dtype=io, bc=bc, seed=3))


@pytest.mark.parametrize("drop", ["z", "D", "delta_bias", "all"])
def test_optional_inputs(ref, drop):
    x = inputs(2, 64, 512, seed=4)
    for k in (("z", "D", "delta_bias") if drop == "all" else (drop,)):
        x[k] = None
    both(ref, x)


def test_softplus_off(ref):
    x = inputs(2, 64, 512, seed=5)
    x["delta"] = (x["delta"].float().abs() * 0.05).to(x["delta"].dtype)   # Delta = delta + bias > 0
    x["delta_bias"] = torch.rand_like(x["delta_bias"]) * 0.05
    both(ref, x, softplus=False)


@pytest.mark.parametrize("K", [2, 5])
def test_segments(ref, K):
    both(ref, inputs(2, 40, 1000, seed=K), num_chunks=K)


def test_two_lane_segments_are_bitwise_single_pass():
    x = inputs(3, 96, 2048, seed=30)
    a, la = run(x, num_chunks=1)
    for K in (2, 8, 64):
        b, lb = run(x, num_chunks=K)
        assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("flags", [0, ONE], ids=["two", "one"])
def test_plain_loads_bitwise_equal_tma(flags):
    x = inputs(2, 96, 512, seed=14)
    a, la = run(x, flags=flags)
    b, lb = run(x, flags=flags | ops.MAMBA_FLAG_NO_TMA)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_start_state(ref):
    x = inputs(2, 64, 512, dtype=torch.float32, seed=8)
    g = torch.Generator(device=DEV)
    g.manual_seed(9)
    h0 = torch.randn(2, 64, 16, generator=g, device=DEV)
    c = {k: (None if v is None else v.cpu()) for k, v in x.items()}
    o_out, o_last = ref.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], D=c["D"],
                                       z=c["z"], delta_bias=c["delta_bias"],
                                       initial_state=h0.cpu())
    for flags in (0, ONE):
        out, last = run(x, flags=flags, initial_state=h0)
        assert max_rel_err(out, o_out) <= tol_for(torch.float32)
        assert max_rel_err(last, o_last) <= tol_for(torch.float32)


def test_one_lane_bounded_wait_reports_timeout():
    x = inputs(1, 64, 1024, seed=33)
    ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], num_chunks=4,
                           flags=ops.MAMBA_FLAG_TEST_WITHHOLD_HANDOFF | ONE)
    torch.cuda.synchronize()
    assert ops.device_status() == -6
    assert ops.device_status() == 0
    out, _ = run(x, num_chunks=4, flags=ONE)
    assert torch.isfinite(out.float()).all()


def test_full_1p4b_layer_kernels_agree():
    """The 1.4B-layer shape (8 x 4096 x 2048, two lanes per channel by
    default): the two kernels agree to bf16 rounding of the output; the
    two-lane one is held to the oracle on sampled chains in test_gpu_scan."""
    c = I.SCAN_CONFIGS["mamba_1p4b_layer"]
    x = I.make_scan_inputs(c, DEV, seed=2)
    assert lanes_of(x) == 2
    a, la = run(x)
    b, lb = run(x, flags=ONE)
    assert max_rel_err(a, b) <= tol_for(torch.bfloat16)
    assert max_rel_err(la, lb) <= 1e-5
