"""Scan over host buffers (mamba_selective_scan_fwd_host): the chunked,
copy-overlapped pipeline against the float64 oracle and against the
device-buffer call, for several chunk sizes (ragged last chunk, more chunks
than the three stages), pinned and pageable memory, a start state, the
zero-order hold, an empty sequence and calls issued back to back."""
import pytest
import torch

from oracle import oracle
from parity import FP32_TOL, max_rel_err, tol_for
from selective_state_space_55_b200 import inputs as I
from selective_state_space_55_b200 import ops

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def ref():
    return oracle.default()


def host_inputs(batch, dim, L, dtype=torch.bfloat16, seed=0, pin=True):
    cfg = I.SCAN_CONFIGS["mamba_1p4b_layer"].resized(batch=batch, dim=dim, seqlen=L,
                                                       io_dtype=dtype, bc_dtype=dtype)
    x = I.make_scan_inputs(cfg, "cpu", seed)
    if pin:
        x = {k: (None if v is None else v.pin_memory()) for k, v in x.items()}
    return x


def run_host(x, **kw):
    res = ops.selective_scan_fwd_host(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"],
                                      z=x["z"], delta_bias=x["delta_bias"],
                                      return_last_state=True, **kw)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    return res


def run_oracle(ref, x, **kw):
    return ref.selective_scan(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                              delta_bias=x["delta_bias"], **kw)


@pytest.mark.parametrize("rows", [0, 1, 3, 8, 20], ids=lambda r: f"rows{r}")
def test_host_chunks_match_oracle_and_device_call(ref, rows):
    x = host_inputs(8, 256, 1024, seed=1)
    out, last = run_host(x, rows=rows)
    o_out, o_last = run_oracle(ref, x)
    assert max_rel_err(out, o_out) <= tol_for(torch.bfloat16)
    assert max_rel_err(last, o_last) <= tol_for(torch.bfloat16)
    xd = {k: (None if v is None else v.to(DEV)) for k, v in x.items()}
    d_out, d_last = ops.selective_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"],
                                           D=xd["D"], z=xd["z"], delta_bias=xd["delta_bias"],
                                           return_last_state=True)
    torch.cuda.synchronize()
    assert max_rel_err(out, d_out.float().cpu().double()) <= tol_for(torch.bfloat16)
    assert max_rel_err(last, d_last.cpu().double()) <= FP32_TOL


def test_pageable_equals_pinned():
    xp = host_inputs(6, 96, 512, seed=2, pin=True)
    xq = {k: (None if v is None else v.clone()) for k, v in xp.items()}   # pageable copies
    assert not xq["u"].is_pinned()
    a_out, a_last = run_host(xp, rows=2)
    out = torch.empty_like(xq["u"])
    last = torch.empty(6, 96, 16)
    b_out, b_last = run_host(xq, rows=2, out=out, last_state=last)
    assert torch.equal(a_out, b_out) and torch.equal(a_last, b_last)


def test_host_fp32_with_start_state_and_zoh(ref):
    x = host_inputs(5, 40, 300, dtype=torch.float32, seed=3)
    g = torch.Generator().manual_seed(4)
    h0 = torch.randn(5, 40, 16, generator=g).pin_memory()
    out, last = run_host(x, rows=2, initial_state=h0, zoh=True)
    o_out, o_last = run_oracle(ref, x, zoh=True, initial_state=h0)
    assert max_rel_err(out, o_out) <= FP32_TOL
    assert max_rel_err(last, o_last) <= FP32_TOL


def test_host_start_state_in_place(ref):
    x = host_inputs(4, 64, 200, dtype=torch.float32, seed=5)
    g = torch.Generator().manual_seed(6)
    h = torch.randn(4, 64, 16, generator=g).pin_memory()
    o_out, o_last = run_oracle(ref, x, initial_state=h.clone())
    out, _ = run_host(x, rows=1, initial_state=h, last_state=h)
    assert max_rel_err(out, o_out) <= FP32_TOL
    assert max_rel_err(h, o_last) <= FP32_TOL


def test_host_empty_sequence_copies_start_state():
    x = host_inputs(3, 24, 0, dtype=torch.float32, seed=7)
    h0 = torch.randn(3, 24, 16).pin_memory()
    last = torch.full((3, 24, 16), float("nan")).pin_memory()
    run_host(x, rows=1, initial_state=h0, last_state=last)
    assert torch.equal(last, h0)


def test_host_calls_back_to_back(ref):
    """Three calls enqueued without synchronising in between (stages and events
    reused across calls) each produce their own correct result."""
    xs = [host_inputs(6, 64, 256, seed=10 + i) for i in range(3)]
    outs = []
    for x in xs:
        outs.append(ops.selective_scan_fwd_host(x["u"], x["delta"], x["A"], x["B"], x["C"],
                                                D=x["D"], z=x["z"], delta_bias=x["delta_bias"],
                                                return_last_state=True, rows=1))
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    for x, (out, last) in zip(xs, outs):
        o_out, o_last = run_oracle(ref, x)
        assert max_rel_err(out, o_out) <= tol_for(torch.bfloat16)
        assert max_rel_err(last, o_last) <= tol_for(torch.bfloat16)


def test_host_workspace_too_small_is_rejected():
    x = host_inputs(2, 32, 64, seed=8)
    need = ops.scan_host_workspace_bytes(2, 32, 16, 64, rows=1)
    ws = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(ops.MambaError, match="WORKSPACE"):
        ops.selective_scan_fwd_host(x["u"], x["delta"], x["A"], x["B"], x["C"], rows=1,
                                    workspace=ws)
