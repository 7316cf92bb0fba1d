"""The scan entry point that allocates nothing (GPU).

Some callers cannot allocate device memory: their device memory belongs to
another allocator that forbids outside cudaMalloc calls, or they run where the
cost and synchronisation of cudaMalloc/cudaFree are not acceptable.  For them
``mamba_selective_scan_fwd_noalloc`` runs the scan with its scratch in a static
8 MiB device array instead of a caller workspace.

These tests call it through the C ABI and check that:
  * its output and last state match ``mamba_selective_scan_fwd`` with a
    caller workspace, on two calls in a row (the shared array keeps the
    previous call's contents, so each call must clear what starts at zero);
  * a problem needing more scratch than the array holds is refused with
    MAMBA_ERR_TOO_LARGE before anything runs.
"""
import ctypes

import pytest
import torch

from parity import max_rel_err, tol_for
from selective_state_space_55_b200 import build
from selective_state_space_55_b200 import inputs as I
from selective_state_space_55_b200 import ops

pytestmark = pytest.mark.gpu

DEV = "cuda"
SCRATCH_BYTES = 8 << 20
MAMBA_ERR_TOO_LARGE = -7
PAR = ops.MAMBA_FLAG_PARALLEL_CHUNKS


def noalloc_fn():
    build.build()
    fn = ops.library().mamba_selective_scan_fwd_noalloc
    vp = ctypes.c_void_p
    fn.restype = ctypes.c_int
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp, vp,
                   ctypes.POINTER(ops.MambaDims), vp]
    return fn


def call_noalloc(x, out, last, num_chunks=0, flags=0):
    batch, dim, L = x["u"].shape
    N = x["A"].shape[1]
    dims = ops.make_scan_dims(batch, dim, N, L, x["u"].dtype, x["B"].dtype, num_chunks, flags)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return noalloc_fn()(p(x["u"]), p(x["delta"]), p(x["A"]), p(x["B"]), p(x["C"]), p(x["D"]),
                        p(x["z"]), p(x["delta_bias"]), 1, p(out), p(last), ctypes.byref(dims),
                        stream)


CASES = {
    # name: (config, overrides, num_chunks, flags)
    "tiny_fp32": ("tiny_fp32", {}, 0, 0),
    "layer_automatic": ("mamba_1p4b_layer", dict(batch=2, dim=512, seqlen=1024), 0, 0),
    "layer_chained_segments": ("mamba_1p4b_layer", dict(batch=4, dim=1024, seqlen=2048), 4, 0),
    "long_parallel_segments": ("long_dna_1m", dict(dim=64, seqlen=8192), 6, PAR),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_workspace_entry_point(name):
    cfg_name, over, K, flags = CASES[name]
    cfg = I.SCAN_CONFIGS[cfg_name].resized(**over)
    x = I.make_scan_inputs(cfg, DEV, seed=7)
    assert ops.scan_workspace_bytes(cfg.batch, cfg.dim, cfg.dstate, cfg.seqlen, cfg.io_dtype,
                                    cfg.bc_dtype, K, flags) <= SCRATCH_BYTES
    want_out, want_last = ops.selective_scan_fwd(
        x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
        delta_bias=x["delta_bias"], return_last_state=True, num_chunks=K, flags=flags)
    torch.cuda.synchronize()
    tol = tol_for(cfg.io_dtype)
    for _ in range(2):
        out = torch.full_like(x["u"], float("nan"))
        last = torch.full((cfg.batch, cfg.dim, cfg.dstate), float("nan"), device=DEV)
        assert call_noalloc(x, out, last, K, flags) == 0
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        assert max_rel_err(out, want_out) <= tol
        assert max_rel_err(last, want_last) <= tol


def test_noalloc_refuses_problems_beyond_its_scratch():
    # Chained segments keep 64 bytes of carry per chain: 64 x 4096 chains need
    # 16 MiB, twice what the array holds.  The call must refuse before it
    # touches any buffer, so these placeholder pointers are never used; u and
    # delta are NULL, so that even a call that got past the size check would
    # stop at the argument check (MAMBA_ERR_INVALID_ARG) before any launch.
    batch, dim, L = 64, 4096, 4096
    assert ops.scan_workspace_bytes(batch, dim, 16, L, num_chunks=2) > SCRATCH_BYTES
    dims = ops.make_scan_dims(batch, dim, 16, L, torch.bfloat16, torch.bfloat16, 2, 0)
    fake = ctypes.c_void_p(0x10000)
    rc = noalloc_fn()(None, None, fake, fake, fake, None, None, None, 1, fake, None,
                      ctypes.byref(dims), None)
    assert rc == MAMBA_ERR_TOO_LARGE
    assert ops.status_string(rc) == "MAMBA_ERR_TOO_LARGE"
