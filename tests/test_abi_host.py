"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol the header declares, plans scans as documented and rejects bad
arguments before touching the device."""
import ctypes
import re
from pathlib import Path

import pytest
import torch

from selective_state_space_55_b200 import build, ops
from selective_state_space_55_b200.inputs import SCAN_CONFIGS

ROOT = Path(__file__).resolve().parent.parent
HEADER = ROOT / "include" / "mamba_ssm.h"
FAKE = ctypes.c_void_p(0x10000)        # never dereferenced: validation fails first


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.library()


def declared_symbols():
    text = HEADER.read_text()
    return re.findall(r"MAMBA_API\s+[\w\s\*]+?\b(mamba_\w+)\s*\(", text)


def test_header_declares_entry_points():
    syms = declared_symbols()
    for name in ("mamba_selective_scan_fwd", "mamba_selective_state_update",
                 "mamba_selective_scan_fwd_with_state", "mamba_selective_scan_fwd_noalloc",
                 "mamba_selective_scan_workspace_bytes", "mamba_selective_scan_plan",
                 "mamba_status_string", "mamba_device_status", "mamba_version"):
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} not exported"


def test_status_strings(lib):
    for code, name in ops.STATUS_NAMES.items():
        assert ops.status_string(code) == name
    assert ops.status_string(-99) == "MAMBA_ERR_UNKNOWN"


def _dims(**kw):
    base = dict(batch=2, dim=64, dstate=16, seqlen=128, io_dtype=torch.bfloat16,
                bc_dtype=torch.bfloat16)
    base.update(kw)
    return ops.make_scan_dims(**base)


def _scan(lib, dims, u=FAKE, delta=FAKE, A=FAKE, B=FAKE, C=FAKE, out=FAKE, D=None, z=None,
          bias=None, last=None):
    return lib.mamba_selective_scan_fwd(u, delta, A, B, C, D, z, bias, 1, out, last,
                                        ctypes.byref(dims) if dims is not None else None, None)


def test_scan_rejects_bad_arguments(lib):
    assert _scan(lib, None) == -1
    assert _scan(lib, _dims(batch=-1)) == -1
    assert _scan(lib, _dims(seqlen=-5)) == -1
    assert _scan(lib, _dims(dstate=0)) == -2
    assert _scan(lib, _dims(dstate=17)) == -2
    d = _dims(); d.io_dtype = 7
    assert _scan(lib, d) == -2
    d = _dims(); d.num_chunks = -1
    assert _scan(lib, d) == -1
    assert _scan(lib, _dims(), u=None) == -1
    assert _scan(lib, _dims(), out=None) == -1
    assert _scan(lib, _dims(), A=None) == -1
    assert _scan(lib, _dims(), C=None) == -1
    # bf16 tensors must be 2-byte aligned, fp32 tensors 4-byte aligned
    assert _scan(lib, _dims(), u=ctypes.c_void_p(0x10001)) == -3
    assert _scan(lib, _dims(), A=ctypes.c_void_p(0x10002)) == -3
    assert _scan(lib, _dims(io_dtype=torch.float32), out=ctypes.c_void_p(0x10002)) == -3


def _scan_h0(lib, dims, h0, last, u=FAKE):
    return lib.mamba_selective_scan_fwd_with_state(u, FAKE, FAKE, FAKE, FAKE, None, None, None, 1,
                                                   h0, FAKE, last, ctypes.byref(dims), None)


def test_scan_with_state_rejects_bad_start_state(lib):
    d = _dims(batch=2, dim=64, dstate=16)            # 2 * 64 * 16 fp32 = 8 KiB of state
    nbytes = 2 * 64 * 16 * 4
    base = 0x100000
    # misaligned start state
    assert _scan_h0(lib, d, ctypes.c_void_p(base + 2), ctypes.c_void_p(base + 0x10000)) == -3
    # partial overlap with last_state, either way round, by one element or by most of it
    for shift in (4, nbytes - 4, -4, -(nbytes - 4)):
        assert _scan_h0(lib, d, ctypes.c_void_p(base), ctypes.c_void_p(base + shift)) == -1
    # the same buffer (in-place continuation) passes these checks and then fails on
    # the null input pointer, still before any device work
    assert _scan_h0(lib, d, ctypes.c_void_p(base), ctypes.c_void_p(base), u=None) == -1
    # disjoint buffers likewise
    assert _scan_h0(lib, d, ctypes.c_void_p(base), ctypes.c_void_p(base + nbytes), u=None) == -1
    # the start-state entry point validates dims like the plain one
    assert _scan_h0(lib, _dims(dstate=17), ctypes.c_void_p(base), None) == -2


def test_host_scan_rejects_bad_arguments(lib):
    d = _dims()
    call = lambda dims, rows, u=FAKE, A=FAKE, out=FAKE: lib.mamba_selective_scan_fwd_host(  # noqa: E731
        u, FAKE, A, FAKE, FAKE, None, None, None, 1, None, out, None, rows,
        ctypes.byref(dims) if dims is not None else None, None)
    assert call(None, 0) == -1
    assert call(d, -1) == -1                      # negative chunk size
    assert call(d, 0, u=None) == -1               # missing input
    assert call(d, 0, A=None) == -1
    assert call(d, 0, out=None) == -1
    assert call(_dims(dstate=17), 0) == -2
    assert call(_dims(batch=0), 0) == 0           # empty problem: nothing to do
    assert lib.mamba_selective_scan_host_workspace_bytes(ctypes.byref(d), -1) == \
        ctypes.c_size_t(-1).value


def test_conv_rejects_bad_arguments(lib):
    d = _dims()
    fwd = lambda dims, W, x=FAKE, w=FAKE, out=FAKE, init=None, fin=None: lib.mamba_causal_conv1d_fwd(  # noqa: E731
        x, w, None, init, W, 1, out, fin, ctypes.byref(dims) if dims is not None else None, None)
    upd = lambda dims, W, st=FAKE, x=FAKE, w=FAKE, out=FAKE: lib.mamba_causal_conv1d_update(  # noqa: E731
        st, x, w, None, W, 1, out, ctypes.byref(dims) if dims is not None else None, None)
    assert fwd(None, 4) == -1
    assert fwd(d, 0) == -2 and fwd(d, 5) == -2          # width outside 1..4
    assert fwd(d, 4, x=None) == -1 and fwd(d, 4, w=None) == -1 and fwd(d, 4, out=None) == -1
    assert fwd(d, 4, x=ctypes.c_void_p(0x10001)) == -3   # bf16 needs 2-byte alignment
    assert fwd(d, 4, out=FAKE, x=FAKE) == -1            # out aliases x
    base = 0x200000
    assert fwd(d, 4, x=ctypes.c_void_p(0x400000), init=ctypes.c_void_p(base),
               fin=ctypes.c_void_p(base + 2)) == -1     # states partly overlap
    bad = _dims(); bad.io_dtype = 9
    assert fwd(bad, 4) == -2
    assert fwd(_dims(batch=0), 4) == 0
    assert upd(None, 4) == -1 and upd(d, 7) == -2
    assert upd(d, 4, st=None) == -1 and upd(d, 4, w=None) == -1
    assert upd(d, 4, w=ctypes.c_void_p(0x10002)) == -3  # fp32 weights need 4-byte alignment


def test_backward_rejects_bad_arguments(lib):
    d = _dims()
    call = lambda dims, u=FAKE, A=FAKE, dout=FAKE, du=FAKE, dA=FAKE: lib.mamba_selective_scan_bwd(  # noqa: E731
        u, FAKE, A, FAKE, FAKE, None, None, None, 1, None, dout, None, du, FAKE, dA, FAKE, FAKE,
        None, None, None, None, ctypes.byref(dims) if dims is not None else None, None)
    assert call(None) == -1
    assert call(_dims(dstate=17)) == -2
    zoh = _dims(); zoh.flags = ops.MAMBA_FLAG_ZOH
    assert call(zoh, u=None) == -1 and call(zoh, A=None) == -1   # the zero-order hold is
    assert call(zoh, u=ctypes.c_void_p(0x10001)) == -3           # checked like Euler
    assert call(d, u=None) == -1 and call(d, dout=None) == -1 and call(d, du=None) == -1
    assert call(d, A=None) == -1 and call(d, dA=None) == -1
    assert call(d, u=ctypes.c_void_p(0x10001)) == -3
    assert call(_dims(batch=0)) == 0


def test_scan_empty_batch_is_a_no_op(lib):
    assert _scan(lib, _dims(batch=0)) == 0
    assert _scan(lib, _dims(dim=0)) == 0


def test_update_rejects_bad_arguments(lib):
    def call(dims, state=FAKE, x=FAKE, out=FAKE):
        return lib.mamba_selective_state_update(state, x, FAKE, FAKE, FAKE, FAKE, None, None,
                                                None, out, ctypes.byref(dims), None)
    good = ops.MambaDims(batch=4, dim=8, dstate=16, io_dtype=1, bc_dtype=1, dt_softplus=1)
    assert call(ops.MambaDims(batch=4, dim=8, dstate=0, io_dtype=1, bc_dtype=1)) == -2
    assert call(ops.MambaDims(batch=-4, dim=8, dstate=16, io_dtype=1, bc_dtype=1)) == -1
    assert call(good, state=None) == -1
    assert call(good, out=None) == -1
    assert call(good, state=ctypes.c_void_p(0x10002)) == -3
    assert call(ops.MambaDims(batch=0, dim=8, dstate=16, io_dtype=1, bc_dtype=1)) == 0


def test_plan_layer_shapes(lib):
    # 2.8B layer: 2560 groups of 32 channels, chained 256-step segments,
    # at most one warp per group
    c = SCAN_CONFIGS["mamba_2p8b_layer"]
    p = ops.scan_plan(c.batch, c.dim, c.dstate, c.seqlen, c.io_dtype, c.bc_dtype)
    assert p["mode"] == 0 and p["launches"] == 1 and p["channels_per_lane"] == 1
    assert p["groups"] == c.batch * c.dim // 32
    assert p["tile_len"] == 16 and p["tma_capable"] == 1
    assert p["nchunks"] == 8 and p["chunk_len"] == 256
    assert p["units_pass_a"] == p["groups"] * 8 and p["units_pass_b"] == 0
    assert p["max_warps"] == min(p["groups"], 148 * 16)
    chains = c.batch * c.dim
    flags = (p["groups"] * 4 + 255) // 256 * 256
    assert p["workspace_bytes"] == 256 + flags + chains * 64
    assert p["lanes_per_channel"] == 1
    # 1.4B layer: 1024 groups of 32 would leave half the 2368 warp slots idle,
    # so each channel gets two lanes: 2048 groups of 16, one warp each, of
    # which the two-lane kernel (12 warps per SM) holds 1776 at once
    c = SCAN_CONFIGS["mamba_1p4b_layer"]
    p = ops.scan_plan(c.batch, c.dim, c.dstate, c.seqlen, c.io_dtype, c.bc_dtype)
    assert p["mode"] == 0 and p["lanes_per_channel"] == 2 and p["groups"] == 2048
    assert p["nchunks"] == 4 and p["max_warps"] == 148 * 12
    assert p["workspace_bytes"] == 256 + 8192 + 8 * 4096 * 64
    q = ops.scan_plan(c.batch, c.dim, c.dstate, c.seqlen, c.io_dtype, c.bc_dtype,
                      flags=ops.MAMBA_FLAG_ONE_LANE_PER_CHANNEL)
    assert q["lanes_per_channel"] == 1 and q["groups"] == 1024 and q["max_warps"] == 1024
    assert q["workspace_bytes"] == 256 + 4096 + 8 * 4096 * 64


def test_plan_two_lanes_per_channel_rules(lib):
    bf = torch.bfloat16
    two = lambda *a, **k: ops.scan_plan(*a, **k)["lanes_per_channel"] == 2  # noqa: E731
    assert two(8, 4096, 16, 2048, bf, bf)                    # chained, 1024 < 2368 groups
    assert not two(16, 5120, 16, 2048, bf, bf)               # 2560 groups fill the GPU
    assert not two(8, 4096, 16, 2048, bf, bf, flags=ops.MAMBA_FLAG_ZOH)
    assert not two(8, 4096, 16, 2048, bf, bf, flags=ops.MAMBA_FLAG_LAYOUT_BLD)
    assert not two(1, 1536, 16, 1 << 20, bf, bf)             # parallel mode
    assert two(1, 64, 16, 100, bf, bf)                       # one short segment, chained
    assert two(2, 100, 16, 512, torch.float32, torch.float32)
    p = ops.scan_plan(3, 40, 16, 4096, bf, bf, num_chunks=4)
    assert p["lanes_per_channel"] == 2 and p["groups"] == 3 * 3 and p["nchunks"] == 4
    p = ops.scan_plan(3, 40, 16, 4096, bf, bf, num_chunks=4, flags=ops.MAMBA_FLAG_PARALLEL_CHUNKS)
    assert p["lanes_per_channel"] == 1 and p["mode"] == 1


def test_plan_parallel_for_the_million_token_sequence(lib):
    # few channel groups: every segment runs at once from its own start (one
    # segment per resident warp), then the carry scan and the correction pass
    # (mode 1), or each segment looks back at the earlier ones and corrects
    # itself in the same launch (mode 2)
    c = SCAN_CONFIGS["long_dna_1m"]
    p = ops.scan_plan(c.batch, c.dim, c.dstate, c.seqlen, c.io_dtype, c.bc_dtype, sm_count=148)
    p2 = ops.scan_plan(c.batch, c.dim, c.dstate, c.seqlen, c.io_dtype, c.bc_dtype, sm_count=148,
                       flags=ops.MAMBA_FLAG_PARALLEL_ONE_LAUNCH)
    K = p["nchunks"]
    assert p2["mode"] == 2 and p2["launches"] == 1 and p2["nchunks"] == K
    assert p2["units_pass_a"] == p["units_pass_a"] and p2["units_pass_b"] == p["units_pass_b"]
    chains = c.batch * c.dim
    flags2 = (K * p["groups"] * 4 + 255) // 256 * 256
    assert p2["workspace_bytes"] == 256 + flags2 + (K * chains * 64 + 255) // 256 * 256 + \
        (K * chains * 4 + 255) // 256 * 256
    assert p["mode"] == 1 and p["launches"] == 3 and p["channels_per_lane"] == 1
    assert p["groups"] == 1536 // 32
    assert K == (148 * 16) // p["groups"]                 # one segment per resident warp
    assert p["units_pass_a"] == p["groups"] * K <= 148 * 16
    assert p["chunk_len"] % p["tile_len"] == 0
    assert (K - 1) * p["chunk_len"] < c.seqlen <= K * p["chunk_len"]
    chains = c.batch * c.dim
    assert p["units_pass_b"] == chains * (K - 1)           # one correction item per later segment
    expect = 256 + 256 + (K * chains * 64 + 255) // 256 * 256 + \
        (K * chains * 4 + 255) // 256 * 256
    assert p["workspace_bytes"] == expect
    assert p["workspace_bytes"] <= 8 << 20


def test_plan_tiny_is_one_segment(lib):
    c = SCAN_CONFIGS["tiny_fp32"]
    p = ops.scan_plan(c.batch, c.dim, c.dstate, c.seqlen, c.io_dtype, c.bc_dtype)
    assert p["nchunks"] == 1 and p["mode"] == 0 and p["tile_len"] == 8
    assert p["workspace_bytes"] == 512


@pytest.mark.parametrize("L,K,want_k,want_len", [
    (100, 5, 4, 32),        # segment length rounds up to the 16-step tile
    (1000, 3, 3, 336),
    (64, 8, 4, 16),
    (31, 4, 2, 16),
    (15, 4, 1, 15),         # shorter than a tile: one segment
])
def test_plan_forced_chunk_counts(lib, L, K, want_k, want_len):
    p = ops.scan_plan(1, 32, 16, L, torch.bfloat16, torch.bfloat16, num_chunks=K)
    assert p["nchunks"] == want_k and p["chunk_len"] == want_len
    assert p["mode"] == 0
    q = ops.scan_plan(1, 32, 16, L, torch.bfloat16, torch.bfloat16, num_chunks=K,
                      flags=ops.MAMBA_FLAG_PARALLEL_CHUNKS)
    assert q["nchunks"] == want_k and q["mode"] == (1 if want_k > 1 else 0)
    q = ops.scan_plan(1, 32, 16, L, torch.bfloat16, torch.bfloat16, num_chunks=K,
                      flags=ops.MAMBA_FLAG_PARALLEL_CHUNKS | ops.MAMBA_FLAG_PARALLEL_ONE_LAUNCH)
    assert q["nchunks"] == want_k and q["mode"] == (2 if want_k > 1 else 0)


def test_plan_tma_capability_follows_strides(lib):
    assert ops.scan_plan(1, 32, 16, 40, torch.bfloat16, torch.bfloat16)["tma_capable"] == 1
    assert ops.scan_plan(1, 32, 16, 37, torch.bfloat16, torch.bfloat16)["tma_capable"] == 0
    assert ops.scan_plan(1, 32, 16, 44, torch.float32, torch.float32)["tma_capable"] == 1
    assert ops.scan_plan(1, 32, 16, 42, torch.float32, torch.float32)["tma_capable"] == 0
    assert ops.scan_plan(1, 32, 16, 44, torch.float32, torch.bfloat16)["tma_capable"] == 0


def test_plan_rejects_bad_dims(lib):
    with pytest.raises(ops.MambaError):
        ops.scan_plan(1, 32, 17, 64)
    with pytest.raises(ops.MambaError):
        ops.scan_plan(-1, 32, 16, 64)


def _ssd(lib, dims, x=FAKE, dt=FAKE, A=FAKE, B=FAKE, C=FAKE, out=FAKE):
    return lib.mamba_ssd_chunk_scan_fwd(x, dt, A, B, C, None, None, None, None, out, None,
                                        ctypes.byref(dims) if dims is not None else None, None)


def _ssd_dims(**kw):
    base = dict(batch=2, seqlen=256, nheads=8, headdim=64, ngroups=1, dstate=128,
                io_dtype=ops.MAMBA_BF16, dt_softplus=1)
    base.update(kw)
    return ops.SsdDims(**base)


def test_ssd_rejects_bad_arguments_before_launch(lib):
    assert _ssd(lib, None) == -1
    assert _ssd(lib, _ssd_dims(batch=-1)) == -1
    assert _ssd(lib, _ssd_dims(seqlen=-1)) == -1
    assert _ssd(lib, _ssd_dims(nheads=6, ngroups=4)) == -1          # groups must divide heads
    assert _ssd(lib, _ssd_dims(headdim=32)) == -2
    assert _ssd(lib, _ssd_dims(dstate=64)) == -2
    assert _ssd(lib, _ssd_dims(io_dtype=ops.MAMBA_F32)) == -2
    assert _ssd(lib, _ssd_dims(), x=None) == -1
    assert _ssd(lib, _ssd_dims(), A=None) == -1
    assert _ssd(lib, _ssd_dims(), out=None) == -1
    assert _ssd(lib, _ssd_dims(), x=ctypes.c_void_p(0x10008)) == -3  # 16-byte rows
    assert _ssd(lib, _ssd_dims(), dt=ctypes.c_void_p(0x10001)) == -3
    assert _ssd(lib, _ssd_dims(batch=0)) == 0                         # nothing to do


def test_ssd_binding_checks_tensors_on_the_host():
    """The Python binding refuses host tensors and wrong shapes or dtypes before
    calling the library (no GPU needed)."""
    x = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
    dt = torch.zeros(1, 8, 2, dtype=torch.bfloat16)
    A = torch.zeros(2)
    B = torch.zeros(1, 8, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        ops.ssd_chunk_scan_fwd(x, dt, A, B, B)


def test_plan_bld_layout(lib):
    """Activations in (batch, seqlen, dim): always chained, TMA when a row of
    channels is a multiple of 16 bytes (and B/C rows are), and the parallel
    mode refused when forced."""
    BLD = ops.MAMBA_FLAG_LAYOUT_BLD
    c = SCAN_CONFIGS["long_dna_1m"]
    p = ops.scan_plan(c.batch, c.dim, c.dstate, c.seqlen, c.io_dtype, c.bc_dtype, flags=BLD)
    assert p["mode"] == 0 and p["launches"] == 1 and p["units_pass_b"] == 0
    assert p["nchunks"] == min((8 * 148 * 16 + p["groups"] - 1) // p["groups"], c.seqlen // 256)
    # TMA needs dim * size (not seqlen * size) to be a multiple of 16 bytes; B/C
    # rows (seqlen * size) still do
    assert ops.scan_plan(1, 40, 16, 40, torch.bfloat16, torch.bfloat16, flags=BLD)["tma_capable"] == 1
    assert ops.scan_plan(1, 36, 16, 40, torch.bfloat16, torch.bfloat16, flags=BLD)["tma_capable"] == 0
    assert ops.scan_plan(1, 40, 16, 37, torch.bfloat16, torch.bfloat16, flags=BLD)["tma_capable"] == 0
    assert ops.scan_plan(1, 40, 16, 40, torch.float32, torch.float32, flags=BLD)["tma_capable"] == 1
    assert ops.scan_plan(1, 38, 16, 40, torch.float32, torch.float32, flags=BLD)["tma_capable"] == 0
    dims = _dims(seqlen=1024)
    dims.num_chunks = 4
    dims.flags = BLD | ops.MAMBA_FLAG_PARALLEL_CHUNKS
    plan = ops.ScanPlan()
    assert lib.mamba_selective_scan_plan(ctypes.byref(dims), 148, ctypes.byref(plan)) == -2
    dims.flags = BLD
    assert lib.mamba_selective_scan_plan(ctypes.byref(dims), 148, ctypes.byref(plan)) == 0


def test_backward_checks_bld_layout_like_the_standard_one(lib):
    d = _dims()
    d.flags = ops.MAMBA_FLAG_LAYOUT_BLD
    call = lambda u=FAKE, dout=FAKE: lib.mamba_selective_scan_bwd(  # noqa: E731
        u, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, None, dout, None, FAKE, FAKE, FAKE, FAKE,
        FAKE, None, None, None, None, ctypes.byref(d), None)
    assert call(u=None) == -1 and call(dout=None) == -1
    assert call(u=ctypes.c_void_p(0x10001)) == -3


def test_binding_layout_argument():
    with pytest.raises(ValueError):
        ops._layout_flags("bdl_", 0)
    assert ops._layout_flags("bld", ops.MAMBA_FLAG_ZOH) == (ops.MAMBA_FLAG_ZOH | ops.MAMBA_FLAG_LAYOUT_BLD, True)
    assert ops._layout_flags("bdl", 0) == (0, False)
    u = torch.empty(2, 7, 5)
    assert ops._scan_sizes(u, True) == (2, 5, 7) and ops._scan_sizes(u, False) == (2, 7, 5)


def test_no_cpu_fallback(tmp_path, lib):
    """A missing library is an error, and host tensors are refused rather
    than computed on the CPU."""
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        ops.library(tmp_path / "absent.so")
    c = SCAN_CONFIGS["tiny_fp32"]
    u = torch.zeros(c.batch, c.dim, c.seqlen)
    A = -torch.ones(c.dim, c.dstate)
    B = torch.zeros(c.batch, c.dstate, c.seqlen)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.selective_scan_fwd(u, u, A, B, B)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.selective_scan_bwd(u, u, A, B, B, u)
