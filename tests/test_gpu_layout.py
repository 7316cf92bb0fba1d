"""Scan forward with activations in the (batch, seqlen, dim) layout
(MAMBA_FLAG_LAYOUT_BLD), the layout of the sample module in
"超越注意力：探索Mamba与状态空间模型", section 代码实现概览.

The kernel runs the same per-channel arithmetic in either layout, so its
outputs must equal the (batch, dim, seqlen) call's bit for bit once transposed;
the float64 oracle (which takes (batch, dim, seqlen)) checks the values on
top, on inputs transposed on the host; the backward likewise.  Cases cover the TMA tiles and the
plain-load path (dim * element size not a multiple of 16 bytes, or
MAMBA_FLAG_NO_TMA), a channel count that leaves a partial group, a ragged
last tile, the optional inputs, the zero-order hold, a start state, and the
full 2.8B-layer shape."""
import pytest
import torch

from oracle import oracle
from parity import FP32_TOL, max_rel_err, tol_for
from selective_state_space_55_b200 import inputs as I
from selective_state_space_55_b200 import ops

pytestmark = pytest.mark.gpu

DEV = "cuda"
ACT = ("u", "delta", "z")
ONE = ops.MAMBA_FLAG_ONE_LANE_PER_CHANNEL


@pytest.fixture(scope="module")
def ref():
    return oracle.default()


def layer_inputs(batch, dim, L, dtype=torch.bfloat16, seed=0, N=16):
    cfg = I.SCAN_CONFIGS["mamba_1p4b_layer"].resized(batch=batch, dim=dim, seqlen=L, dstate=N,
                                                       io_dtype=dtype, bc_dtype=dtype,
                                                       recipe="layer")
    return I.make_scan_inputs(cfg, DEV, seed)


def to_bld(t):
    return None if t is None else t.transpose(1, 2).contiguous()


def scan(x, layout, **kw):
    args = {k: (to_bld(x[k]) if layout == "bld" else x[k]) for k in ACT}
    out, last = ops.selective_scan_fwd(args["u"], args["delta"], x["A"], x["B"], x["C"],
                                       D=x["D"], z=args["z"], delta_bias=x["delta_bias"],
                                       return_last_state=True, layout=layout, **kw)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    if layout == "bld":
        assert out.shape == args["u"].shape
        out = out.transpose(1, 2)
    return out, last


def oracle_scan(ref, x, **kw):
    c = lambda t: None if t is None else t.cpu()  # noqa: E731
    return ref.selective_scan(c(x["u"]), c(x["delta"]), c(x["A"]), c(x["B"]), c(x["C"]),
                              D=c(x["D"]), z=c(x["z"]), delta_bias=c(x["delta_bias"]), **kw)


def check(ref, x, tol, zoh=False, h0=None, flags=0):
    """Bitwise against the (batch, dim, seqlen) call with one lane per channel
    (the kernel this layout runs) in one segment (chained segments reproduce it
    bit for bit), and within tol of the oracle."""
    out_b, last_b = scan(x, "bld", zoh=zoh, initial_state=h0, flags=flags)
    out_d, last_d = scan(x, "bdl", zoh=zoh, initial_state=h0, num_chunks=1, flags=ONE)
    assert torch.equal(out_b, out_d)
    assert torch.equal(last_b, last_d)
    o_out, o_last = oracle_scan(ref, x, zoh=zoh, initial_state=None if h0 is None else h0.cpu())
    e_out, e_last = max_rel_err(out_b, o_out), max_rel_err(last_b, o_last)
    assert e_out <= tol, f"out error {e_out:.3e} > {tol:.1e}"
    assert e_last <= tol, f"last_state error {e_last:.3e} > {tol:.1e}"


def test_tiny_fp32(ref):
    x = I.make_scan_inputs(I.SCAN_CONFIGS["tiny_fp32"], DEV, seed=0)
    check(ref, x, FP32_TOL)


@pytest.mark.parametrize("dtype,shape", [
    (torch.bfloat16, (2, 256, 2048)),    # TMA tiles, whole groups
    (torch.float32, (2, 96, 1024)),
    (torch.bfloat16, (3, 200, 1000)),    # partial group of 8 channels, ragged last tile
    (torch.float32, (2, 36, 777)),       # odd L: B/C rows unaligned, plain loads
    (torch.bfloat16, (2, 100, 512)),     # 200-byte rows of steps: plain loads
    (torch.bfloat16, (1, 8, 96)),        # fewer channels than a group
])
def test_layer_recipe(ref, dtype, shape):
    x = layer_inputs(*shape, dtype=dtype, seed=11)
    check(ref, x, tol_for(dtype))


@pytest.mark.parametrize("opt", ["no_z", "no_D", "no_bias", "plain"])
def test_optional_inputs(ref, opt):
    x = layer_inputs(2, 128, 640, seed=3)
    if opt in ("no_z", "plain"):
        x["z"] = None
    if opt in ("no_D", "plain"):
        x["D"] = None
    if opt in ("no_bias", "plain"):
        x["delta_bias"] = None
    check(ref, x, tol_for(torch.bfloat16))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_plain_loads_bitwise_equal_tma(dtype):
    x = layer_inputs(2, 160, 1024, dtype=dtype, seed=4)
    a = scan(x, "bld")
    b = scan(x, "bld", flags=ops.MAMBA_FLAG_NO_TMA)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_zero_order_hold(ref):
    x = layer_inputs(2, 128, 1024, seed=6)
    check(ref, x, tol_for(torch.bfloat16), zoh=True)


def test_start_state(ref):
    x = layer_inputs(2, 96, 512, dtype=torch.float32, seed=7)
    g = torch.Generator(device=DEV)
    g.manual_seed(8)
    h0 = torch.randn(2, 96, 16, generator=g, device=DEV)
    check(ref, x, FP32_TOL, h0=h0)


def test_few_channels_long_sequence_runs_chained(ref):
    """(batch, dim, seqlen) would take the parallel mode here; the
    (batch, seqlen, dim) call stays chained and matches the oracle."""
    x = layer_inputs(1, 64, 16384, seed=9)
    plan = ops.scan_plan(1, 64, 16, 16384, flags=ops.MAMBA_FLAG_LAYOUT_BLD)
    assert plan["mode"] == 0 and ops.scan_plan(1, 64, 16, 16384)["mode"] != 0
    out, last = scan(x, "bld")
    o_out, o_last = oracle_scan(ref, x)
    assert max_rel_err(out, o_out) <= tol_for(torch.bfloat16)
    assert max_rel_err(last, o_last) <= tol_for(torch.bfloat16)


def test_full_2p8b_layer_bitwise():
    """The 2.8B-layer shape (16 x 5120 channels x 2048 steps): the
    (batch, seqlen, dim) call equals the (batch, dim, seqlen) one bit for bit;
    the latter is held to the oracle on sampled chains elsewhere."""
    c = I.SCAN_CONFIGS["mamba_2p8b_layer"]
    x = I.make_scan_inputs(c, DEV, seed=1)
    a = scan(x, "bld")
    b = scan(x, "bdl", flags=ONE)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_host_buffer_call():
    x = layer_inputs(4, 128, 512, seed=12)
    dev_out, dev_last = scan(x, "bld")
    h = {k: (None if v is None else v.cpu().pin_memory()) for k, v in x.items()}
    out, last = ops.selective_scan_fwd_host(to_bld(h["u"]).pin_memory(),
                                            to_bld(h["delta"]).pin_memory(), h["A"], h["B"],
                                            h["C"], D=h["D"], z=to_bld(h["z"]).pin_memory(),
                                            delta_bias=h["delta_bias"], return_last_state=True,
                                            rows=3, layout="bld")
    torch.cuda.synchronize()
    assert torch.equal(out.transpose(1, 2), dev_out.cpu())
    assert torch.equal(last, dev_last.cpu())


def test_parallel_chunks_are_refused():
    x = layer_inputs(1, 64, 1024, seed=2)
    with pytest.raises(ops.MambaError):
        scan(x, "bld", num_chunks=4, flags=ops.MAMBA_FLAG_PARALLEL_CHUNKS)


# ------------------------------------------------------------ backward

def backward(x, dout, layout, zoh=False, h0=None, dlast=None, softplus=True):
    args = {k: (to_bld(x[k]) if layout == "bld" else x[k]) for k in ACT}
    g = ops.selective_scan_bwd(args["u"], args["delta"], x["A"], x["B"], x["C"],
                               to_bld(dout) if layout == "bld" else dout, D=x["D"], z=args["z"],
                               delta_bias=x["delta_bias"], initial_state=h0, dlast_state=dlast,
                               zoh=zoh, layout=layout, softplus=softplus)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    if layout == "bld":
        for k in ("du", "ddelta", "dz"):
            if k in g:
                g[k] = g[k].transpose(1, 2)
    return g


@pytest.mark.parametrize("dtype,shape,zoh", [
    (torch.bfloat16, (2, 256, 1000), False),   # staged tiles, ragged last block
    (torch.float32, (2, 96, 512), False),
    (torch.bfloat16, (3, 200, 777), False),    # a partial last group: read directly
    (torch.bfloat16, (2, 100, 300), False),    # 200-byte rows of channels: read directly
    (torch.bfloat16, (2, 128, 640), True),
])
def test_backward_matches_standard_layout(dtype, shape, zoh):
    """Per-chain gradients (du, ddelta, dz) are the same arithmetic in either
    layout and equal bit for bit; the gradients summed over chains (dA, dB,
    dC, dD, the bias) are added atomically in no fixed order and agree to
    rounding."""
    x = layer_inputs(*shape, dtype=dtype, seed=21)
    g = torch.Generator(device=DEV)
    g.manual_seed(22)
    dout = torch.randn(*shape, generator=g, device=DEV).to(dtype)
    h0 = torch.randn(shape[0], shape[1], 16, generator=g, device=DEV)
    dlast = torch.randn(shape[0], shape[1], 16, generator=g, device=DEV)
    a = backward(x, dout, "bld", zoh=zoh, h0=h0, dlast=dlast)
    b = backward(x, dout, "bdl", zoh=zoh, h0=h0, dlast=dlast)
    assert set(a) == set(b)
    for k in ("du", "ddelta", "dz", "dinitial_state"):
        assert torch.equal(a[k], b[k]), k
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        assert max_rel_err(a[k], b[k]) <= 1e-5, k


@pytest.mark.parametrize("case", ["layer", "N4", "softplus_off", "plain", "zoh_start_state"])
def test_backward_against_oracle(ref, case):
    """fp32 inputs in (batch, seqlen, dim): every gradient against the
    oracle (which takes (batch, dim, seqlen)), over the options: a state of 4
    entries, softplus off (delta kept positive), no gate, D or bias, and the
    zero-order hold from a start state with a last-state gradient."""
    N = 4 if case == "N4" else 16
    x = layer_inputs(2, 64, 300, dtype=torch.float32, seed=23, N=N)
    softplus = case != "softplus_off"
    if not softplus:
        x["delta"] = x["delta"].abs() * 0.05
        x["delta_bias"] = torch.full_like(x["delta_bias"], 0.01)
    if case == "plain":
        x["z"] = x["D"] = x["delta_bias"] = None
    g = torch.Generator(device=DEV)
    g.manual_seed(24)
    dout = torch.randn(2, 64, 300, generator=g, device=DEV)
    zoh = case == "zoh_start_state"
    h0 = torch.randn(2, 64, N, generator=g, device=DEV) if zoh else None
    dlast = torch.randn(2, 64, N, generator=g, device=DEV) if zoh else None
    got = backward(x, dout, "bld", zoh=zoh, h0=h0, dlast=dlast, softplus=softplus)
    c = lambda t: None if t is None else t.cpu()  # noqa: E731
    o = ref.selective_scan_bwd(c(x["u"]), c(x["delta"]), c(x["A"]), c(x["B"]), c(x["C"]), dout.cpu(),
                               D=c(x["D"]), z=c(x["z"]), delta_bias=c(x["delta_bias"]),
                               softplus=softplus, initial_state=c(h0), dlast_state=c(dlast), zoh=zoh)
    assert set(got) == set(o), (set(got), set(o))
    for k in o:
        assert max_rel_err(got[k], o[k]) <= FP32_TOL, k
