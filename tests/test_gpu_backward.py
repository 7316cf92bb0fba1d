"""Backward pass of the scan (mamba_selective_scan_bwd): every gradient against
the float64 oracle's adjoint, which finite differences of the forward oracle
pin.  fp32 and bf16, with and without gate / D / bias / softplus / start
state / last-state gradient, state sizes below 16, ragged lengths and channel
counts, sequences cut into many chained segments, and all of it again with
the zero-order-hold input term.  At the benchmark's full size (the 2.8B layer
shape): sampled chains and channels against the oracle, and the two
activation layouts against each other."""
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


def problem(batch, dim, L, dtype=torch.float32, N=16, seed=0, gated=True):
    cfg = I.SCAN_CONFIGS["mamba_1p4b_layer"].resized(batch=batch, dim=dim, seqlen=L, dstate=N,
                                                       io_dtype=dtype, bc_dtype=dtype)
    x = I.make_scan_inputs(cfg, DEV, seed)
    g = torch.Generator(device=DEV)
    g.manual_seed(seed + 99)
    x["dout"] = torch.randn(batch, dim, L, generator=g, device=DEV).to(dtype)
    x["h0"] = torch.randn(batch, dim, N, generator=g, device=DEV) if gated else None
    x["dlast"] = torch.randn(batch, dim, N, generator=g, device=DEV) if gated else None
    if not gated:
        x["z"] = x["D"] = x["delta_bias"] = None
    return x


def check(ref, x, tol, softplus=True, zoh=False, **kw):
    g = ops.selective_scan_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dout"], D=x["D"],
                               z=x["z"], delta_bias=x["delta_bias"], softplus=softplus,
                               initial_state=x["h0"], dlast_state=x["dlast"], zoh=zoh, **kw)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    c = lambda t: None if t is None else t.cpu()  # noqa: E731
    o = ref.selective_scan_bwd(c(x["u"]), c(x["delta"]), c(x["A"]), c(x["B"]), c(x["C"]),
                               c(x["dout"]), D=c(x["D"]), z=c(x["z"]), delta_bias=c(x["delta_bias"]),
                               softplus=softplus, initial_state=c(x["h0"]), dlast_state=c(x["dlast"]),
                               zoh=zoh)
    assert set(g) == set(o), (set(g), set(o))
    errs = {k: max_rel_err(g[k], o[k]) for k in o}
    bad = {k: e for k, e in errs.items() if e > tol}
    assert not bad, f"gradients beyond {tol:.0e}: {bad}"
    return errs


def test_fp32_all_gradients(ref):
    check(ref, problem(2, 70, 300, seed=1), FP32_TOL)


def test_fp32_plain(ref):
    """No gate, D, bias, start state or last-state gradient; softplus off (Delta =
    delta itself, drawn positive so that the state decays)."""
    x = problem(2, 40, 200, seed=2, gated=False)
    x["delta"] = x["delta"].abs() * 0.1
    check(ref, x, FP32_TOL, softplus=False)


@pytest.mark.parametrize("N", [1, 5, 8])
def test_state_sizes(ref, N):
    check(ref, problem(1, 33, 130, N=N, seed=3 + N), FP32_TOL)


@pytest.mark.parametrize("L", [1, 7, 8, 9, 257])
def test_ragged_lengths(ref, L):
    check(ref, problem(2, 32, L, seed=10 + L), FP32_TOL)


def test_many_segments(ref):
    """Few chains and a long sequence: 16 chained segments hand lambda backwards."""
    check(ref, problem(1, 64, 4096, seed=20), FP32_TOL)


def test_bf16_layer_recipe(ref):
    check(ref, problem(2, 256, 2048, dtype=torch.bfloat16, seed=21), BF16_TOL)


def test_last_state_gradient_only(ref):
    """dout = 0: every gradient flows from dlast_state through the adjoint alone."""
    x = problem(2, 48, 333, seed=22)
    x["dout"] = torch.zeros_like(x["dout"])
    check(ref, x, FP32_TOL)


def test_unaligned_rows_take_scalar_path(ref):
    """A length whose rows are not 16-byte aligned (L * 4 % 16 != 0)."""
    check(ref, problem(2, 36, 301, seed=23), FP32_TOL)


# ---- zero-order-hold input term (MAMBA_FLAG_ZOH)

def test_zoh_fp32_all_gradients(ref):
    check(ref, problem(2, 70, 300, seed=31), FP32_TOL, zoh=True)


def test_zoh_fp32_plain(ref):
    x = problem(2, 40, 200, seed=32, gated=False)
    x["delta"] = x["delta"].abs() * 0.1
    check(ref, x, FP32_TOL, softplus=False, zoh=True)


def test_zoh_small_and_zero_A(ref):
    """Entries of A at 0 (the gain's limit Delta) and near 0, where dg/dA takes
    its series; others across the closed form's range."""
    x = problem(2, 64, 256, seed=33)
    A = x["A"].clone()
    A[:, 0] = 0.0
    A[:, 1] = -1e-3
    A[:, 2] = -0.05
    A[:, 3] = -0.6
    x["A"] = A
    check(ref, x, FP32_TOL, zoh=True)


@pytest.mark.parametrize("N", [1, 5, 16])
def test_zoh_state_sizes(ref, N):
    check(ref, problem(1, 33, 130, N=N, seed=34 + N), FP32_TOL, zoh=True)


def test_zoh_many_segments(ref):
    check(ref, problem(1, 64, 4096, seed=35), FP32_TOL, zoh=True)


def test_zoh_bf16_layer_recipe(ref):
    check(ref, problem(2, 256, 2048, dtype=torch.bfloat16, seed=36), BF16_TOL, zoh=True)


# ------------------------------------------------------------ full size

def full_size_backward(layout="bdl"):
    """The backward's benchmark workload: the 2.8B layer shape (16 x 5120
    channels x 2048 steps, bf16), gate, D and bias on, dout random."""
    cfg = I.SCAN_CONFIGS["mamba_2p8b_layer"]
    x = I.make_scan_inputs(cfg, DEV, seed=0)
    g = torch.Generator(device=DEV)
    g.manual_seed(13)
    dout = torch.randn(cfg.batch, cfg.dim, cfg.seqlen, generator=g, device=DEV).to(cfg.io_dtype)
    act = {k: x[k] for k in ("u", "delta", "z")}
    dy = dout
    if layout == "bld":
        act = {k: v.transpose(1, 2).contiguous() for k, v in act.items()}
        dy = dout.transpose(1, 2).contiguous()
    grads = ops.selective_scan_bwd(act["u"], act["delta"], x["A"], x["B"], x["C"], dy, D=x["D"],
                                   z=act["z"], delta_bias=x["delta_bias"], layout=layout)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    if layout == "bld":
        for k in ("du", "ddelta", "dz"):
            grads[k] = grads[k].transpose(1, 2)
    return cfg, x, dout, grads


def test_full_size_sampled_chains_and_channels(ref):
    """du, delta's gradient and dz of a chain depend only on that chain and
    its batch row's B and C, so sampled chains are checked against the oracle
    run on each alone; dA, dD and the bias gradient of a channel sum over the
    batch rows, so sampled channels are checked against the oracle run on that
    channel over all 16 rows.  (dB and dC sum over all 5120 channels; the
    smaller cases above check them.)"""
    cfg, x, dout, g = full_size_backward()
    for row in I.gather_chains(x, I.sample_chains(cfg.batch, cfg.dim, 8, seed=5)):
        b, d = row["b"], row["d"]
        o = ref.selective_scan_bwd(row["u"], row["delta"], row["A"], row["B"], row["C"],
                                   dout[b:b + 1, d:d + 1].cpu(), D=row["D"], z=row["z"],
                                   delta_bias=row["delta_bias"])
        for k in ("du", "ddelta", "dz"):
            e = max_rel_err(g[k][b:b + 1, d:d + 1], o[k])
            assert e <= BF16_TOL, f"chain ({b},{d}) {k} error {e:.3e}"
    for d in (0, 2047, cfg.dim - 1):
        c = lambda t: t[:, d:d + 1].cpu()  # noqa: E731
        o = ref.selective_scan_bwd(c(x["u"]), c(x["delta"]), x["A"][d:d + 1].cpu(), x["B"].cpu(),
                                   x["C"].cpu(), c(dout), D=x["D"][d:d + 1].cpu(), z=c(x["z"]),
                                   delta_bias=x["delta_bias"][d:d + 1].cpu())
        assert max_rel_err(g["dA"][d:d + 1], o["dA"]) <= BF16_TOL, f"channel {d} dA"
        assert max_rel_err(g["dD"][d:d + 1], o["dD"]) <= BF16_TOL, f"channel {d} dD"
        assert max_rel_err(g["ddelta_bias"][d:d + 1], o["ddelta_bias"]) <= BF16_TOL, f"channel {d} bias"


def test_full_size_layouts_agree():
    """The same workload with activations in (batch, seqlen, dim): the
    per-chain gradients equal the (batch, dim, seqlen) call's bit for bit; the
    sums over chains (atomics in no fixed order) agree to rounding."""
    a = full_size_backward("bdl")[3]
    b = full_size_backward("bld")[3]
    for k in ("du", "ddelta", "dz"):
        assert torch.equal(a[k], b[k]), k
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        assert max_rel_err(a[k], b[k]) <= 1e-4, k
