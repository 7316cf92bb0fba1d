"""Short causal convolution (prefill and decode update): CUDA path through the C
ABI vs the float64 oracle.  Widths 1..4, both dtypes, the 16-byte vector path
and the any-length path (ragged lengths, L < W, L = 0), initial and final conv
state (also one buffer for both), bias and silu on and off, updates against the
prefill, and the Mamba-2.8B layer and decode shapes."""
import pytest
import torch

from oracle import oracle
from parity import FP32_TOL, max_rel_err, tol_for
from selective_state_space_55_b200 import ops

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def ref():
    return oracle.default()


def conv_inputs(batch, dim, L, W, dtype, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    x = torch.randn(batch, dim, L, generator=g, device=DEV).to(dtype)
    w = torch.randn(dim, W, generator=g, device=DEV) / W
    bias = torch.randn(dim, generator=g, device=DEV)
    init = torch.randn(batch, dim, W, generator=g, device=DEV).to(dtype)
    return x, w, bias, init


def c(t):
    return None if t is None else t.cpu()


@pytest.mark.parametrize("L", [2048, 1000, 999, 40, 3, 1])
@pytest.mark.parametrize("W", [1, 2, 3, 4])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_prefill_matches_oracle(ref, dtype, W, L):
    x, w, bias, init = conv_inputs(2, 96, L, W, dtype, seed=W * 1000 + L)
    out, final = ops.causal_conv1d_fwd(x, w, bias=bias, initial_conv_state=init,
                                       return_final_state=True)
    torch.cuda.synchronize()
    o_out, o_final = ref.causal_conv1d(c(x), c(w), bias=c(bias), initial_conv_state=c(init))
    assert max_rel_err(out, o_out) <= tol_for(dtype)
    assert max_rel_err(final, o_final) == 0.0


@pytest.mark.parametrize("silu", [True, False])
def test_prefill_options(ref, silu):
    x, w, _, _ = conv_inputs(3, 40, 512, 4, torch.float32, seed=7)
    out = ops.causal_conv1d_fwd(x, w, silu=silu)          # no bias, zero start
    torch.cuda.synchronize()
    o_out, _ = ref.causal_conv1d(c(x), c(w), silu=silu)
    assert max_rel_err(out, o_out) <= FP32_TOL


def test_prefill_empty_sequence_keeps_state():
    x, w, bias, init = conv_inputs(2, 24, 0, 4, torch.bfloat16, seed=8)
    _, final = ops.causal_conv1d_fwd(x, w, bias=bias, initial_conv_state=init,
                                     return_final_state=True)
    torch.cuda.synchronize()
    assert torch.equal(final, init)


def test_prefill_state_in_place(ref):
    x, w, bias, init = conv_inputs(2, 64, 2, 4, torch.float32, seed=9)   # L < W
    st = init.clone()
    out, _ = ops.causal_conv1d_fwd(x, w, bias=bias, initial_conv_state=st, final_conv_state=st)
    torch.cuda.synchronize()
    o_out, o_final = ref.causal_conv1d(c(x), c(w), bias=c(bias), initial_conv_state=c(init))
    assert max_rel_err(out, o_out) <= FP32_TOL
    assert max_rel_err(st, o_final) == 0.0


def test_prefill_layer_shape(ref):
    """Mamba-2.8B layer shape (5120 channels, L 2048, W 4, bf16), 4 batch rows."""
    x, w, bias, init = conv_inputs(4, 5120, 2048, 4, torch.bfloat16, seed=10)
    out, final = ops.causal_conv1d_fwd(x, w, bias=bias, return_final_state=True)
    torch.cuda.synchronize()
    o_out, o_final = ref.causal_conv1d(c(x), c(w), bias=c(bias))
    assert max_rel_err(out, o_out) <= tol_for(torch.bfloat16)
    assert max_rel_err(final, o_final) == 0.0


@pytest.mark.parametrize("W", [1, 2, 3, 4])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_update_matches_oracle(ref, dtype, W):
    x, w, bias, init = conv_inputs(8, 320, 1, W, dtype, seed=20 + W)
    xt = x[:, :, 0].contiguous()
    st = init.clone()
    out = ops.causal_conv1d_update(st, xt, w, bias=bias)
    torch.cuda.synchronize()
    o_st, o_out = ref.causal_conv1d_update(c(init), c(xt), c(w), bias=c(bias))
    assert max_rel_err(st, o_st) == 0.0
    assert max_rel_err(out, o_out) <= tol_for(dtype)


def test_update_misaligned_state_uses_generic_path(ref):
    """A state that starts 2 bytes off its 8-byte boundary takes the scalar path."""
    x, w, bias, init = conv_inputs(4, 64, 1, 4, torch.bfloat16, seed=30)
    buf = torch.empty(init.numel() + 1, dtype=torch.bfloat16, device=DEV)
    st = buf[1:].view(init.shape)
    st.copy_(init)
    xt = x[:, :, 0].contiguous()
    out = ops.causal_conv1d_update(st, xt, w, bias=bias)
    torch.cuda.synchronize()
    o_st, o_out = ref.causal_conv1d_update(c(init), c(xt), c(w), bias=c(bias))
    assert max_rel_err(st, o_st) == 0.0
    assert max_rel_err(out, o_out) <= tol_for(torch.bfloat16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_updates_continue_prefill(dtype):
    """Prefill over T1 tokens, then updates over the rest, equals one prefill."""
    x, w, bias, init = conv_inputs(3, 128, 40, 4, dtype, seed=31)
    out_all, final_all = ops.causal_conv1d_fwd(x, w, bias=bias, initial_conv_state=init,
                                               return_final_state=True)
    T1 = 17
    _, st = ops.causal_conv1d_fwd(x[:, :, :T1].contiguous(), w, bias=bias,
                                  initial_conv_state=init, return_final_state=True)
    outs = [ops.causal_conv1d_update(st, x[:, :, t].contiguous(), w, bias=bias)
            for t in range(T1, 40)]
    torch.cuda.synchronize()
    assert max_rel_err(torch.stack(outs, dim=-1), out_all[:, :, T1:].double()) <= tol_for(dtype)
    assert torch.equal(st, final_all)


def test_update_decode_shape(ref):
    """Decode shape: batch 128 x 4096 channels, W 4, bf16 state."""
    x, w, bias, init = conv_inputs(128, 4096, 1, 4, torch.bfloat16, seed=32)
    xt = x[:, :, 0].contiguous()
    st = init.clone()
    out = ops.causal_conv1d_update(st, xt, w, bias=bias)
    torch.cuda.synchronize()
    o_st, o_out = ref.causal_conv1d_update(c(init), c(xt), c(w), bias=c(bias))
    assert max_rel_err(st, o_st) == 0.0
    assert max_rel_err(out, o_out) <= tol_for(torch.bfloat16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_update_ragged_chain_count(ref, dtype):
    """15 chains: three quads take the 4-chains-per-thread path, the last 3 its tail."""
    x, w, bias, init = conv_inputs(3, 5, 1, 4, dtype, seed=33)
    xt = x[:, :, 0].contiguous()
    st = init.clone()
    out = ops.causal_conv1d_update(st, xt, w, bias=bias)
    torch.cuda.synchronize()
    o_st, o_out = ref.causal_conv1d_update(c(init), c(xt), c(w), bias=c(bias))
    assert max_rel_err(st, o_st) == 0.0
    assert max_rel_err(out, o_out) <= tol_for(dtype)


def test_update_one_chain_per_thread_path(ref):
    """A bf16 state 8-byte but not 16-byte aligned takes the one-chain vector path."""
    x, w, bias, init = conv_inputs(4, 64, 1, 4, torch.bfloat16, seed=34)
    buf = torch.empty(init.numel() + 4, dtype=torch.bfloat16, device=DEV)
    st = buf[4:].view(init.shape)
    assert st.data_ptr() % 16 == 8
    st.copy_(init)
    xt = x[:, :, 0].contiguous()
    out = ops.causal_conv1d_update(st, xt, w, bias=bias)
    torch.cuda.synchronize()
    o_st, o_out = ref.causal_conv1d_update(c(init), c(xt), c(w), bias=c(bias))
    assert max_rel_err(st, o_st) == 0.0
    assert max_rel_err(out, o_out) <= tol_for(torch.bfloat16)


def test_update_dependent_launch_is_bitwise_identical():
    """MAMBA_FLAG_PDL on the W = 4 decode update (each layer's launch may start
    while the previous layer's finishes; the layers' conv states are distinct):
    the same states and outputs bit for bit as plain launches, over 48 layers x
    3 tokens inside a CUDA graph."""
    g = torch.Generator(device=DEV)
    g.manual_seed(91)
    L, batch, dim = 48, 8, 512
    base = [torch.randn(batch, dim, 4, generator=g, device=DEV).to(torch.bfloat16) for _ in range(L)]
    xs = [[torch.randn(batch, dim, generator=g, device=DEV).to(torch.bfloat16) for _ in range(L)]
          for _ in range(3)]
    ws = [torch.randn(dim, 4, generator=g, device=DEV) for _ in range(L)]
    bs = [torch.randn(dim, generator=g, device=DEV) for _ in range(L)]
    results = []
    for flags in (0, ops.MAMBA_FLAG_PDL):
        states = [b.clone() for b in base]
        outs = [[torch.empty_like(x) for x in row] for row in xs]
        graphs = []
        for t in range(3):
            keep = [st.clone() for st in states]
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for i in range(L):
                    ops.causal_conv1d_update(states[i], xs[t][i], ws[i], bias=bs[i],
                                             out=outs[t][i], flags=flags)
            for st, k in zip(states, keep):
                st.copy_(k)
            graphs.append(graph)
        for graph in graphs:
            graph.replay()
        torch.cuda.synchronize()
        results.append((states, outs))
    (s0, o0), (s1, o1) = results
    for a, b in zip(s0, s1):
        assert torch.equal(a, b)
    for ra, rb in zip(o0, o1):
        for a, b in zip(ra, rb):
            assert torch.equal(a, b)
