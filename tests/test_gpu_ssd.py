"""Mamba-2 layer (scalar A per head) on the tensor cores: CUDA path through the C
ABI vs the float64 oracle's recurrence.  Every case must meet both gates: the
max relative error of ``parity.max_rel_err`` at most ``BF16_TOL`` (2e-2, bf16
inputs with the fp32 state) on the output and on the final state, and the
componentwise bound of ``parity.SCALED_TOL`` (error at most 2^-8 of the summed
term magnitudes).  The final state, which the kernel keeps in fp32 and builds
from hi/lo operand pairs, is further held to 1e-3 (``FINAL_STATE_TOL``): a
single bf16 rounding of the weighted input would leave it near 1.5e-2.

Cases: the small three-chunk workload (ragged last chunk, two groups, start
state), every optional input off in turn, lengths at and around the chunk
boundary, the start state alone (x = 0, which isolates the chunk-entry product),
a sequence scanned in two calls, an empty sequence, and the Mamba-2 2.7B layer
shape checked on sampled (batch, head) chains against the oracle run on those
chains alone."""
import numpy as np
import pytest
import torch

from oracle import oracle
from parity import BF16_TOL, SCALED_TOL, max_rel_err, max_scaled_err
from selective_state_space_55_b200 import ops
from selective_state_space_55_b200.inputs import SSD_CONFIGS, make_ssd_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"
FINAL_STATE_TOL = 1e-3


@pytest.fixture(scope="module")
def ref():
    return oracle.default()


def cpu(p):
    return {k: (None if v is None else v.cpu()) for k, v in p.items()}


def run_gpu(p, softplus=True):
    out, final = ops.ssd_chunk_scan_fwd(p["x"], p["dt"], p["A"], p["B"], p["C"], D=p["D"],
                                        z=p["z"], dt_bias=p["dt_bias"], dt_softplus=softplus,
                                        initial_state=p["initial_state"],
                                        return_final_state=True)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    return out, final


def run_ref(ref, p, softplus=True):
    c = cpu(p)
    return ref.ssd_scan(c["x"], c["dt"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                        dt_bias=c["dt_bias"], dt_softplus=softplus,
                        initial_state=c["initial_state"])


def magnitude(ref, p, softplus=True):
    """Per element, the sum of the magnitudes of the terms that reach it: the
    recurrence on |x|, |B|, |C|, |D|, |start state| (the decay factors are
    positive), times |silu(z)|; the same for the final state."""
    c = cpu(p)
    ab = {k: (None if c[k] is None else c[k].double().abs())
          for k in ("x", "B", "C", "D", "initial_state")}
    y, fin = ref.ssd_scan(ab["x"], c["dt"], c["A"], ab["B"], ab["C"], D=ab["D"], z=None,
                          dt_bias=c["dt_bias"], dt_softplus=softplus,
                          initial_state=ab["initial_state"])
    if c["z"] is not None:
        zz = c["z"].double().numpy()
        y = y * np.abs(zz / (1.0 + np.exp(-zz)))
    return y, fin


def check(ref, p, softplus=True, what=""):
    out, final = run_gpu(p, softplus)
    o_out, o_final = run_ref(ref, p, softplus)
    s_out, s_final = magnitude(ref, p, softplus)
    e_out, e_fin = max_scaled_err(out, o_out, s_out), max_scaled_err(final, o_final, s_final)
    assert e_out <= SCALED_TOL and e_fin <= SCALED_TOL, (what, e_out, e_fin)
    r_out, r_fin = max_rel_err(out, o_out), max_rel_err(final, o_final)
    assert r_out <= BF16_TOL and r_fin <= FINAL_STATE_TOL, (what, r_out, r_fin)
    return r_out, r_fin


def small(**kw):
    return SSD_CONFIGS["ssd_small"].resized(**kw)


def test_small_workload(ref):
    check(ref, make_ssd_inputs(small(), DEV, seed=0), what="ssd_small")


@pytest.mark.parametrize("drop", ["z", "D", "dt_bias", "initial_state"])
def test_optional_inputs_off(ref, drop):
    p = make_ssd_inputs(small(), DEV, seed=1)
    p[drop] = None
    check(ref, p, what=f"without {drop}")


def test_softplus_off(ref):
    p = make_ssd_inputs(small(), DEV, seed=2)
    p["dt"] = (p["dt"].float().abs() * 0.05).to(torch.bfloat16)   # Delta = dt + bias >= 0
    p["dt_bias"] = torch.zeros_like(p["dt_bias"])
    check(ref, p, softplus=False, what="softplus off")


@pytest.mark.parametrize("L", [1, 7, 127, 128, 129, 256, 383])
def test_lengths_around_the_chunk(ref, L):
    check(ref, make_ssd_inputs(small(seqlen=L), DEV, seed=10 + L), what=f"L={L}")


@pytest.mark.parametrize("ngroups", [1, 4])
def test_groups(ref, ngroups):
    check(ref, make_ssd_inputs(small(ngroups=ngroups, nheads=8), DEV, seed=20 + ngroups),
          what=f"ngroups={ngroups}")


def test_start_state_alone(ref):
    """x = 0: the output is the decayed start state read out through C."""
    p = make_ssd_inputs(small(seqlen=200), DEV, seed=3)
    p["x"] = torch.zeros_like(p["x"])
    p["D"] = None
    check(ref, p, what="x = 0")


def test_single_token_state(ref):
    """No start state, one token: the state is Delta x B^T (the chunk-state product)."""
    check(ref, make_ssd_inputs(small(seqlen=1, initial_state=False), DEV, seed=4),
          what="one token")


def test_split_equals_whole(ref):
    cfg = small(seqlen=384)
    p = make_ssd_inputs(cfg, DEV, seed=5)
    out, final = run_gpu(p)
    k = 128
    a = {n: (v[:, :k].contiguous() if n in ("x", "dt", "B", "C", "z") else v)
         for n, v in p.items()}
    b = {n: (v[:, k:].contiguous() if n in ("x", "dt", "B", "C", "z") else v)
         for n, v in p.items()}
    out1, mid = run_gpu(a)
    b["initial_state"] = mid
    out2, final2 = run_gpu(b)
    o_out, o_final = run_ref(ref, p)
    s_out, s_final = magnitude(ref, p)
    joined = torch.cat([out1, out2], dim=1)
    assert max_scaled_err(joined, out.cpu(), s_out) <= SCALED_TOL
    assert max_scaled_err(final2, final.cpu(), s_final) <= SCALED_TOL
    assert max_scaled_err(joined, o_out, s_out) <= SCALED_TOL
    assert max_scaled_err(final2, o_final, s_final) <= SCALED_TOL
    assert max_rel_err(joined, o_out) <= BF16_TOL
    assert max_rel_err(final2, o_final) <= FINAL_STATE_TOL


def test_empty_sequence_keeps_state():
    p = make_ssd_inputs(small(seqlen=0), DEV, seed=6)
    out, final = run_gpu(p)
    assert out.numel() == 0
    assert torch.equal(final, p["initial_state"])
    p["initial_state"] = None
    _, final = run_gpu(p)
    assert torch.count_nonzero(final) == 0


def test_deterministic():
    p = make_ssd_inputs(small(), DEV, seed=7)
    a, fa = run_gpu(p)
    b, fb = run_gpu(p)
    assert torch.equal(a, b) and torch.equal(fa, fb)


def test_mamba2_layer_sampled_chains(ref):
    """Mamba-2 2.7B layer shape; six (batch, head) chains re-run in the oracle."""
    cfg = SSD_CONFIGS["mamba2_2p7b_layer"]
    p = make_ssd_inputs(cfg, DEV, seed=0)
    out, final = run_gpu(p)
    H, G = cfg.nheads, cfg.ngroups
    rng = np.random.default_rng(0)
    picks = {(0, 0), (cfg.batch - 1, H - 1)}
    while len(picks) < 6:
        picks.add((int(rng.integers(cfg.batch)), int(rng.integers(H))))
    for b, h in sorted(picks):
        g = h // (H // G)
        sub = dict(x=p["x"][b:b + 1, :, h:h + 1], dt=p["dt"][b:b + 1, :, h:h + 1],
                   A=p["A"][h:h + 1], B=p["B"][b:b + 1, :, g:g + 1],
                   C=p["C"][b:b + 1, :, g:g + 1], D=p["D"][h:h + 1], z=p["z"][b:b + 1, :, h:h + 1],
                   dt_bias=p["dt_bias"][h:h + 1], initial_state=None)
        o_out, o_final = run_ref(ref, sub)
        s_out, s_final = magnitude(ref, sub)
        e_out = max_scaled_err(out[b:b + 1, :, h:h + 1], o_out, s_out)
        e_fin = max_scaled_err(final[b:b + 1, h:h + 1], o_final, s_final)
        assert e_out <= SCALED_TOL and e_fin <= SCALED_TOL, ((b, h), e_out, e_fin)
        r_out = max_rel_err(out[b:b + 1, :, h:h + 1], o_out)
        r_fin = max_rel_err(final[b:b + 1, h:h + 1], o_final)
        assert r_out <= BF16_TOL and r_fin <= FINAL_STATE_TOL, ((b, h), r_out, r_fin)


def test_rejects_unsupported_shape():
    p = make_ssd_inputs(small(seqlen=16), DEV, seed=8)
    x = torch.zeros(2, 16, 4, 32, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ops.MambaError, match="UNSUPPORTED"):
        ops.ssd_chunk_scan_fwd(x, p["dt"], p["A"], p["B"], p["C"])
