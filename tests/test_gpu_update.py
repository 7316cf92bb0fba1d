"""Single-token state update: CUDA path (through the C ABI) vs the float64 oracle."""
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


def decode_cfg(batch=128, dim=4096, N=16, io=torch.bfloat16, bc=torch.bfloat16):
    return I.DecodeConfig("t", batch=batch, dim=dim, dstate=N, layers=1, steps=1, io_dtype=io,
                          bc_dtype=bc)


def one_step(ref, cfg, layer, tok, dt_softplus=True, state=None):
    state = layer["state"].clone() if state is None else state
    before = state.cpu()
    out = ops.selective_state_update(state, tok["x"], tok["dt"], layer["A"], tok["B"], tok["C"],
                                     D=layer["D"], z=tok["z"], dt_bias=layer["dt_bias"],
                                     dt_softplus=dt_softplus)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    c = lambda t: None if t is None else t.cpu()  # noqa: E731
    o_state, o_out = ref.selective_state_update(
        before, c(tok["x"]), c(tok["dt"]), c(layer["A"]), c(tok["B"]), c(tok["C"]),
        D=c(layer["D"]), z=c(tok["z"]), dt_bias=c(layer["dt_bias"]), dt_softplus=dt_softplus)
    return state, out, o_state, o_out


def test_decode_layer_shape_full_compare(ref):
    cfg = I.DECODE_CONFIG
    layer = I.make_decode_layer(cfg, DEV, seed=1)
    tok = I.make_decode_token(cfg, DEV, seed=2)
    state, out, o_state, o_out = one_step(ref, cfg, layer, tok)
    assert max_rel_err(state, o_state) <= FP32_TOL
    assert max_rel_err(out, o_out) <= BF16_TOL


@pytest.mark.parametrize("io,bc", [(torch.float32, torch.float32), (torch.float32, torch.bfloat16),
                                   (torch.bfloat16, torch.float32)])
def test_decode_dtypes(ref, io, bc):
    cfg = decode_cfg(8, 320, io=io, bc=bc)
    layer = I.make_decode_layer(cfg, DEV, seed=3)
    tok = I.make_decode_token(cfg, DEV, seed=4)
    state, out, o_state, o_out = one_step(ref, cfg, layer, tok)
    assert max_rel_err(state, o_state) <= FP32_TOL
    assert max_rel_err(out, o_out) <= tol_for(io)


@pytest.mark.parametrize("N", [1, 3, 5, 8, 16])
def test_decode_generic_state_sizes(ref, N):
    cfg = decode_cfg(4, 100, N=N, io=torch.float32, bc=torch.float32)
    layer = I.make_decode_layer(cfg, DEV, seed=N)
    tok = I.make_decode_token(cfg, DEV, seed=N + 1)
    state, out, o_state, o_out = one_step(ref, cfg, layer, tok)
    assert max_rel_err(state, o_state) <= FP32_TOL
    assert max_rel_err(out, o_out) <= FP32_TOL


def test_decode_unaligned_state_uses_generic_path(ref):
    cfg = decode_cfg(4, 64, io=torch.float32, bc=torch.float32)
    layer = I.make_decode_layer(cfg, DEV, seed=9)
    tok = I.make_decode_token(cfg, DEV, seed=10)
    buf = torch.empty(4 * 64 * 16 + 1, device=DEV)
    state = buf[1:].view(4, 64, 16)
    state.copy_(layer["state"])
    state, out, o_state, o_out = one_step(ref, cfg, layer, tok, state=state)
    assert max_rel_err(state, o_state) <= FP32_TOL
    assert max_rel_err(out, o_out) <= FP32_TOL


@pytest.mark.parametrize("drop", ["z", "D", "dt_bias", "softplus"])
def test_decode_optional_inputs(ref, drop):
    cfg = decode_cfg(8, 128, io=torch.float32, bc=torch.float32)
    layer = I.make_decode_layer(cfg, DEV, seed=11)
    tok = I.make_decode_token(cfg, DEV, seed=12)
    sp = True
    if drop == "z":
        tok["z"] = None
    elif drop in ("D", "dt_bias"):
        layer[drop] = None
    else:
        sp = False                                # Delta = dt + dt_bias must stay positive
        tok["dt"] = tok["dt"].abs() * 0.1
        layer["dt_bias"] = torch.rand_like(layer["dt_bias"]) * 0.05
    state, out, o_state, o_out = one_step(ref, cfg, layer, tok, dt_softplus=sp)
    assert max_rel_err(state, o_state) <= FP32_TOL
    assert max_rel_err(out, o_out) <= FP32_TOL


def test_decode_leaves_inputs_unchanged():
    cfg = decode_cfg(8, 128)
    layer = I.make_decode_layer(cfg, DEV, seed=13)
    tok = I.make_decode_token(cfg, DEV, seed=14)
    snap = {k: v.clone() for k, v in tok.items()}
    ops.selective_state_update(layer["state"], tok["x"], tok["dt"], layer["A"], tok["B"], tok["C"],
                               D=layer["D"], z=tok["z"], dt_bias=layer["dt_bias"])
    torch.cuda.synchronize()
    for k in snap:
        assert torch.equal(snap[k], tok[k])


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_decode_steps_equal_scan(ref, io):
    """128 updates from the zero state = the scan over the same 128 tokens (GPU and oracle)."""
    batch, dim, N, T = 4, 256, 16, 128
    cfg = I.SCAN_CONFIGS["mamba_1p4b_layer"].resized(batch=batch, dim=dim, seqlen=T, io_dtype=io,
                                                       bc_dtype=io)
    x = I.make_scan_inputs(cfg, DEV, seed=21)
    scan_out, scan_last = ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"],
                                                 D=x["D"], z=x["z"], delta_bias=x["delta_bias"],
                                                 return_last_state=True)
    state = torch.zeros(batch, dim, N, device=DEV)
    outs = torch.empty_like(x["u"])
    for t in range(T):
        outs[:, :, t] = ops.selective_state_update(
            state, x["u"][:, :, t].contiguous(), x["delta"][:, :, t].contiguous(), x["A"],
            x["B"][:, :, t].contiguous(), x["C"][:, :, t].contiguous(), D=x["D"],
            z=x["z"][:, :, t].contiguous(), dt_bias=x["delta_bias"])
    torch.cuda.synchronize()
    cpu = {k: v.cpu() for k, v in x.items()}
    o_out, o_last = ref.selective_scan(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"],
                                       D=cpu["D"], z=cpu["z"], delta_bias=cpu["delta_bias"])
    tol = tol_for(io)
    assert max_rel_err(outs, o_out) <= tol
    assert max_rel_err(state, o_last) <= FP32_TOL
    assert max_rel_err(outs, scan_out.double()) <= tol
    assert max_rel_err(state, scan_last.double()) <= FP32_TOL


def test_decode_48_layers_rotating(ref):
    """The benchmark's pattern: 48 distinct layer states, each updated in turn."""
    cfg = decode_cfg(16, 512)
    layers = [I.make_decode_layer(cfg, DEV, seed=100 + i) for i in range(48)]
    toks = [I.make_decode_token(cfg, DEV, seed=200 + i) for i in range(48)]
    before = [l["state"].cpu() for l in layers]
    outs = []
    for l, t in zip(layers, toks):
        outs.append(ops.selective_state_update(l["state"], t["x"], t["dt"], l["A"], t["B"], t["C"],
                                               D=l["D"], z=t["z"], dt_bias=l["dt_bias"]))
    torch.cuda.synchronize()
    for i in (0, 17, 47):
        l, t = layers[i], toks[i]
        c = lambda v: v.cpu()  # noqa: E731
        o_state, o_out = ref.selective_state_update(before[i], c(t["x"]), c(t["dt"]), c(l["A"]),
                                                    c(t["B"]), c(t["C"]), D=c(l["D"]), z=c(t["z"]),
                                                    dt_bias=c(l["dt_bias"]))
        assert max_rel_err(l["state"], o_state) <= FP32_TOL
        assert max_rel_err(outs[i], o_out) <= BF16_TOL


@pytest.mark.parametrize("dim", [1024, 136, 8])
def test_decode_streaming_and_plain_paths_agree(ref, dim):
    """The bulk-TMA streaming path (dim % 8 == 0, with a partial last tile of the
    128-channel tiles) and the plain-load path both match the oracle."""
    cfg = decode_cfg(6, dim)
    layer = I.make_decode_layer(cfg, DEV, seed=dim)
    tok = I.make_decode_token(cfg, DEV, seed=dim + 1)
    results = []
    for flags in (0, ops.MAMBA_FLAG_NO_TMA):
        state = layer["state"].clone()
        out = ops.selective_state_update(state, tok["x"], tok["dt"], layer["A"], tok["B"],
                                         tok["C"], D=layer["D"], z=tok["z"],
                                         dt_bias=layer["dt_bias"], flags=flags)
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        results.append((state, out))
    c = lambda t: t.cpu()  # noqa: E731
    o_state, o_out = ref.selective_state_update(
        c(layer["state"]), c(tok["x"]), c(tok["dt"]), c(layer["A"]), c(tok["B"]), c(tok["C"]),
        D=c(layer["D"]), z=c(tok["z"]), dt_bias=c(layer["dt_bias"]))
    for state, out in results:
        assert max_rel_err(state, o_state) <= FP32_TOL
        assert max_rel_err(out, o_out) <= BF16_TOL
    assert max_rel_err(results[0][0], results[1][0].double()) <= FP32_TOL


@pytest.mark.parametrize("graph", [False, True], ids=["eager", "cuda_graph"])
def test_decode_dependent_launch_is_bitwise_identical(graph):
    """MAMBA_FLAG_PDL (each layer's launch may start while the previous layer's
    finishes; the layers' states are distinct) gives the same states and outputs
    bit for bit as plain launches, over 48 layers x 3 tokens, eagerly and inside
    a CUDA graph."""
    cfg = decode_cfg(16, 1024)
    L = 48
    base = [I.make_decode_layer(cfg, DEV, seed=500 + i) for i in range(L)]
    toks = [[I.make_decode_token(cfg, DEV, seed=700 + 10 * t + i) for i in range(L)] for t in range(3)]
    results = []
    for flags in (0, ops.MAMBA_FLAG_PDL):
        states = [b["state"].clone() for b in base]
        outs = [[torch.empty_like(tk["x"]) for tk in row] for row in toks]

        def step(t):
            for i in range(L):
                tk, lay = toks[t][i], base[i]
                ops.selective_state_update(states[i], tk["x"], tk["dt"], lay["A"], tk["B"], tk["C"],
                                           D=lay["D"], z=tk["z"], dt_bias=lay["dt_bias"],
                                           out=outs[t][i], flags=flags)

        if graph:
            graphs = []
            for t in range(3):
                s = torch.cuda.Stream()
                s.wait_stream(torch.cuda.current_stream())
                torch.cuda.synchronize()
                g = torch.cuda.CUDAGraph()
                keep = [st.clone() for st in states]
                with torch.cuda.graph(g):
                    step(t)
                for st, k in zip(states, keep):     # capture ran nothing; restore anyway
                    st.copy_(k)
                graphs.append(g)
            for g in graphs:
                g.replay()
        else:
            for t in range(3):
                step(t)
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        results.append((states, outs))
    (s0, o0), (s1, o1) = results
    for a, b in zip(s0, s1):
        assert torch.equal(a, b)
    for ra, rb in zip(o0, o1):
        for a, b in zip(ra, rb):
            assert torch.equal(a, b)
