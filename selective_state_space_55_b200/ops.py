"""Python binding of the C ABI in ``include/mamba_ssm.h`` (ctypes).

Argument marshalling only: tensors are checked for device, dtype and layout,
their data pointers and sizes are packed into ``mamba_dims_t`` and the call
goes to ``libmamba_ssm.so``.  Every step of the computation runs in the
library's CUDA kernels; PyTorch only supplies device memory (including the
scan's scratch workspace) and the current stream.  There is no fallback: if
the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

PKG = Path(__file__).resolve().parent
LIBRARY_PATH = PKG / "libmamba_ssm.so"

MAMBA_OK = 0
STATUS_NAMES = {
    0: "MAMBA_OK", -1: "MAMBA_ERR_INVALID_ARG", -2: "MAMBA_ERR_UNSUPPORTED",
    -3: "MAMBA_ERR_ALIGN", -4: "MAMBA_ERR_WORKSPACE", -5: "MAMBA_ERR_CUDA",
    -6: "MAMBA_ERR_TIMEOUT", -7: "MAMBA_ERR_TOO_LARGE",
}
MAMBA_F32, MAMBA_BF16 = 0, 1
MAMBA_FLAG_NO_TMA = 0x1
MAMBA_FLAG_PARALLEL_CHUNKS = 0x2
MAMBA_FLAG_TEST_WITHHOLD_HANDOFF = 0x4
MAMBA_FLAG_ZOH = 0x8
MAMBA_FLAG_PDL = 0x10
MAMBA_FLAG_LAYOUT_BLD = 0x20
MAMBA_FLAG_ONE_LANE_PER_CHANNEL = 0x40
MAMBA_FLAG_PARALLEL_ONE_LAUNCH = 0x80

_DTYPE_CODE = {torch.float32: MAMBA_F32, torch.bfloat16: MAMBA_BF16}


class MambaDims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64), ("dim", ctypes.c_int64), ("dstate", ctypes.c_int64),
        ("seqlen", ctypes.c_int64), ("io_dtype", ctypes.c_int32), ("bc_dtype", ctypes.c_int32),
        ("dt_softplus", ctypes.c_int32), ("num_chunks", ctypes.c_int32),
        ("flags", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


class SsdDims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
        ("headdim", ctypes.c_int64), ("ngroups", ctypes.c_int64), ("dstate", ctypes.c_int64),
        ("io_dtype", ctypes.c_int32), ("dt_softplus", ctypes.c_int32),
    ]


class ScanPlan(ctypes.Structure):
    _fields_ = [
        ("nchunks", ctypes.c_int32), ("tile_len", ctypes.c_int32),
        ("chunk_len", ctypes.c_int64), ("groups", ctypes.c_int64),
        ("units_pass_a", ctypes.c_int64), ("units_pass_b", ctypes.c_int64),
        ("warps_per_cta", ctypes.c_int32), ("launches", ctypes.c_int32),
        ("tma_capable", ctypes.c_int32), ("mode", ctypes.c_int32),
        ("channels_per_lane", ctypes.c_int32), ("lanes_per_channel", ctypes.c_int32),
        ("max_warps", ctypes.c_int64), ("workspace_bytes", ctypes.c_size_t),
    ]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


class MambaError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        super().__init__(f"{call} failed: {STATUS_NAMES.get(status, status)}")


_LIB = None


def library(path: Path | str | None = None) -> ctypes.CDLL:
    """Load (once) and return the CUDA library; raises if it is missing."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = Path(path) if path is not None else LIBRARY_PATH
    if not p.exists():
        raise RuntimeError(
            f"{p} is missing: build it with `python -m selective_state_space_55_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(str(p))
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    dims_p = ctypes.POINTER(MambaDims)
    lib.mamba_selective_scan_plan.restype = i32
    lib.mamba_selective_scan_plan.argtypes = [dims_p, i32, ctypes.POINTER(ScanPlan)]
    lib.mamba_selective_scan_workspace_bytes.restype = ctypes.c_size_t
    lib.mamba_selective_scan_workspace_bytes.argtypes = [dims_p]
    lib.mamba_selective_scan_fwd.restype = i32
    lib.mamba_selective_scan_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, dims_p, vp]
    lib.mamba_selective_scan_fwd_with_state.restype = i32
    lib.mamba_selective_scan_fwd_with_state.argtypes = [
        vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, dims_p, vp]
    lib.mamba_selective_scan_host_workspace_bytes.restype = ctypes.c_size_t
    lib.mamba_selective_scan_host_workspace_bytes.argtypes = [dims_p, ctypes.c_int64]
    lib.mamba_selective_scan_fwd_host.restype = i32
    lib.mamba_selective_scan_fwd_host.argtypes = [
        vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, ctypes.c_int64, dims_p, vp]
    lib.mamba_selective_scan_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.mamba_selective_scan_bwd_workspace_bytes.argtypes = [dims_p]
    lib.mamba_selective_scan_bwd.restype = i32
    lib.mamba_selective_scan_bwd.argtypes = [vp] * 8 + [i32] + [vp] * 12 + [dims_p, vp]
    lib.mamba_causal_conv1d_fwd.restype = i32
    lib.mamba_causal_conv1d_fwd.argtypes = [vp, vp, vp, vp, i32, i32, vp, vp, dims_p, vp]
    lib.mamba_causal_conv1d_update.restype = i32
    lib.mamba_causal_conv1d_update.argtypes = [vp, vp, vp, vp, i32, i32, vp, dims_p, vp]
    lib.mamba_selective_state_update.restype = i32
    lib.mamba_selective_state_update.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, dims_p, vp]
    lib.mamba_ssd_chunk_scan_fwd.restype = i32
    lib.mamba_ssd_chunk_scan_fwd.argtypes = [vp] * 11 + [ctypes.POINTER(SsdDims), vp]
    lib.mamba_device_status.restype = i32
    lib.mamba_device_status.argtypes = []
    lib.mamba_status_string.restype = ctypes.c_char_p
    lib.mamba_status_string.argtypes = [i32]
    lib.mamba_version.restype = ctypes.c_char_p
    lib.mamba_version.argtypes = []
    if path is None:
        _LIB = lib
    return lib


def status_string(status: int) -> str:
    return library().mamba_status_string(status).decode()


def version() -> str:
    return library().mamba_version().decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_cuda(name, t, dtypes, shape):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_host(name, t, dtypes, shape):
    if t is None:
        return
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream_handle(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _layout_flags(layout, flags):
    """Flags with MAMBA_FLAG_LAYOUT_BLD set for ``layout="bld"``, and whether it is set."""
    if layout not in ("bdl", "bld"):
        raise ValueError(f"layout must be 'bdl' or 'bld', not {layout!r}")
    if layout == "bld":
        flags |= MAMBA_FLAG_LAYOUT_BLD
    return flags, bool(flags & MAMBA_FLAG_LAYOUT_BLD)


def _scan_sizes(u, bld):
    """(batch, dim, L) of the activations u."""
    if u.dim() != 3:
        raise ValueError(f"u must have 3 dimensions, got shape {tuple(u.shape)}")
    if bld:
        batch, L, dim = u.shape
    else:
        batch, dim, L = u.shape
    return batch, dim, L


def make_scan_dims(batch, dim, dstate, seqlen, io_dtype, bc_dtype, num_chunks=0, flags=0,
                   workspace=None) -> MambaDims:
    return MambaDims(batch=batch, dim=dim, dstate=dstate, seqlen=seqlen,
                     io_dtype=_DTYPE_CODE[io_dtype], bc_dtype=_DTYPE_CODE[bc_dtype],
                     dt_softplus=0, num_chunks=num_chunks, flags=flags, reserved=0,
                     workspace=None if workspace is None else workspace.data_ptr(),
                     workspace_bytes=0 if workspace is None else workspace.numel())


def scan_plan(batch, dim, dstate, seqlen, io_dtype=torch.bfloat16, bc_dtype=torch.bfloat16,
              num_chunks=0, sm_count=148, flags=0) -> dict:
    """The library's plan for a scan of these sizes on a GPU with ``sm_count`` SMs."""
    dims = make_scan_dims(batch, dim, dstate, seqlen, io_dtype, bc_dtype, num_chunks, flags)
    plan = ScanPlan()
    rc = library().mamba_selective_scan_plan(ctypes.byref(dims), sm_count, ctypes.byref(plan))
    if rc != MAMBA_OK:
        raise MambaError("mamba_selective_scan_plan", rc)
    return plan.as_dict()


def scan_workspace_bytes(batch, dim, dstate, seqlen, io_dtype=torch.bfloat16,
                         bc_dtype=torch.bfloat16, num_chunks=0, flags=0) -> int:
    """Scratch bytes the scan needs on the current device."""
    dims = make_scan_dims(batch, dim, dstate, seqlen, io_dtype, bc_dtype, num_chunks, flags)
    n = library().mamba_selective_scan_workspace_bytes(ctypes.byref(dims))
    if n == ctypes.c_size_t(-1).value:
        raise MambaError("mamba_selective_scan_workspace_bytes", -1)
    return int(n)


def selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                       out=None, last_state=None, return_last_state=False, num_chunks=0,
                       flags=0, workspace=None, stream=None, initial_state=None, zoh=False,
                       layout="bdl"):
    """Selective scan forward through ``mamba_selective_scan_fwd`` (or
    ``mamba_selective_scan_fwd_with_state`` when ``initial_state`` is given).

    u, delta, z: (batch, dim, L) fp32 or bf16 (one dtype), or (batch, L, dim)
    with ``layout="bld"`` (MAMBA_FLAG_LAYOUT_BLD); B, C: (batch, N, L)
    fp32 or bf16; A: (dim, N) fp32; D, delta_bias: (dim,) fp32 or None;
    initial_state: (batch, dim, N) fp32 start state or None (zero).  ``zoh``
    sets MAMBA_FLAG_ZOH (zero-order-hold input term).
    Returns ``out`` (u's shape and dtype), and the fp32 last state
    (batch, dim, N) too when ``return_last_state`` or ``last_state`` is given.
    """
    flags, bld = _layout_flags(layout, flags)
    batch, dim, L = _scan_sizes(u, bld)
    act = (batch, L, dim) if bld else (batch, dim, L)
    N = A.shape[1]
    io, bc = u.dtype, B.dtype
    _check_cuda("u", u, (torch.float32, torch.bfloat16), act)
    _check_cuda("delta", delta, (io,), act)
    _check_cuda("z", z, (io,), act)
    _check_cuda("A", A, (torch.float32,), (dim, N))
    _check_cuda("B", B, (torch.float32, torch.bfloat16), (batch, N, L))
    _check_cuda("C", C, (bc,), (batch, N, L))
    _check_cuda("D", D, (torch.float32,), (dim,))
    _check_cuda("delta_bias", delta_bias, (torch.float32,), (dim,))
    if out is None:
        out = torch.empty_like(u)
    _check_cuda("out", out, (io,), act)
    if last_state is None and return_last_state:
        last_state = torch.empty((batch, dim, N), dtype=torch.float32, device=u.device)
    _check_cuda("last_state", last_state, (torch.float32,), (batch, dim, N))
    _check_cuda("initial_state", initial_state, (torch.float32,), (batch, dim, N))
    if zoh:
        flags |= MAMBA_FLAG_ZOH
    if workspace is None:
        need = scan_workspace_bytes(batch, dim, N, L, io, bc, num_chunks, flags)
        if need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=u.device)
    dims = make_scan_dims(batch, dim, N, L, io, bc, num_chunks, flags, workspace)
    if initial_state is None:
        name = "mamba_selective_scan_fwd"
        rc = library().mamba_selective_scan_fwd(
            _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
            int(bool(softplus)), _ptr(out), _ptr(last_state), ctypes.byref(dims),
            _stream_handle(stream))
    else:
        name = "mamba_selective_scan_fwd_with_state"
        rc = library().mamba_selective_scan_fwd_with_state(
            _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
            int(bool(softplus)), _ptr(initial_state), _ptr(out), _ptr(last_state),
            ctypes.byref(dims), _stream_handle(stream))
    if rc != MAMBA_OK:
        raise MambaError(name, rc)
    if last_state is not None:
        return out, last_state
    return out


def scan_host_workspace_bytes(batch, dim, dstate, seqlen, io_dtype=torch.bfloat16,
                              bc_dtype=torch.bfloat16, rows=0, num_chunks=0, flags=0) -> int:
    """Device scratch bytes of ``selective_scan_fwd_host`` on the current device."""
    dims = make_scan_dims(batch, dim, dstate, seqlen, io_dtype, bc_dtype, num_chunks, flags)
    n = library().mamba_selective_scan_host_workspace_bytes(ctypes.byref(dims), rows)
    if n == ctypes.c_size_t(-1).value:
        raise MambaError("mamba_selective_scan_host_workspace_bytes", -1)
    return int(n)


def selective_scan_fwd_host(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                            out=None, last_state=None, return_last_state=False, rows=0,
                            num_chunks=0, flags=0, workspace=None, stream=None,
                            initial_state=None, zoh=False, device=None, layout="bdl"):
    """Selective scan over HOST tensors through ``mamba_selective_scan_fwd_host``.

    Every tensor argument is a contiguous CPU tensor (page-locked for the copies
    to overlap the scans), with the shapes and dtypes of ``selective_scan_fwd``.
    ``rows`` batch rows go through the device per chunk (0: automatic).
    ``workspace`` is a device uint8 tensor of at least ``scan_host_workspace_bytes``
    (allocated on ``device``, default the current CUDA device, when None).
    The call returns once the work is enqueued on ``stream``; synchronise it
    before reading ``out`` / ``last_state``.  Returns ``out`` (and the last
    state, as ``selective_scan_fwd`` does).  ``layout`` as for ``selective_scan_fwd``.
    """
    flags, bld = _layout_flags(layout, flags)
    batch, dim, L = _scan_sizes(u, bld)
    act = (batch, L, dim) if bld else (batch, dim, L)
    N = A.shape[1]
    io, bc = u.dtype, B.dtype
    _check_host("u", u, (torch.float32, torch.bfloat16), act)
    _check_host("delta", delta, (io,), act)
    _check_host("z", z, (io,), act)
    _check_host("A", A, (torch.float32,), (dim, N))
    _check_host("B", B, (torch.float32, torch.bfloat16), (batch, N, L))
    _check_host("C", C, (bc,), (batch, N, L))
    _check_host("D", D, (torch.float32,), (dim,))
    _check_host("delta_bias", delta_bias, (torch.float32,), (dim,))
    _check_host("initial_state", initial_state, (torch.float32,), (batch, dim, N))
    pin = torch.cuda.is_available()
    if out is None:
        out = torch.empty(u.shape, dtype=io, pin_memory=pin)
    _check_host("out", out, (io,), act)
    if last_state is None and return_last_state:
        last_state = torch.empty((batch, dim, N), dtype=torch.float32, pin_memory=pin)
    _check_host("last_state", last_state, (torch.float32,), (batch, dim, N))
    if zoh:
        flags |= MAMBA_FLAG_ZOH
    if workspace is None:
        need = scan_host_workspace_bytes(batch, dim, N, L, io, bc, rows, num_chunks, flags)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    dims = make_scan_dims(batch, dim, N, L, io, bc, num_chunks, flags, workspace)
    rc = library().mamba_selective_scan_fwd_host(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        int(bool(softplus)), _ptr(initial_state), _ptr(out), _ptr(last_state), rows,
        ctypes.byref(dims), _stream_handle(stream))
    if rc != MAMBA_OK:
        raise MambaError("mamba_selective_scan_fwd_host", rc)
    if last_state is not None:
        return out, last_state
    return out


def selective_state_update(state, x, dt, A, B, C, D=None, z=None, dt_bias=None,
                           dt_softplus=True, out=None, flags=0, stream=None, zoh=False):
    """One generation step through ``mamba_selective_state_update``; ``state`` is
    updated in place.  ``zoh`` sets MAMBA_FLAG_ZOH.  Returns ``out`` (batch, dim) in
    x's dtype."""
    if zoh:
        flags |= MAMBA_FLAG_ZOH
    batch, dim, N = state.shape
    io, bc = x.dtype, B.dtype
    _check_cuda("state", state, (torch.float32,), (batch, dim, N))
    _check_cuda("x", x, (torch.float32, torch.bfloat16), (batch, dim))
    _check_cuda("dt", dt, (io,), (batch, dim))
    _check_cuda("z", z, (io,), (batch, dim))
    _check_cuda("A", A, (torch.float32,), (dim, N))
    _check_cuda("B", B, (torch.float32, torch.bfloat16), (batch, N))
    _check_cuda("C", C, (bc,), (batch, N))
    _check_cuda("D", D, (torch.float32,), (dim,))
    _check_cuda("dt_bias", dt_bias, (torch.float32,), (dim,))
    if out is None:
        out = torch.empty_like(x)
    _check_cuda("out", out, (io,), (batch, dim))
    dims = MambaDims(batch=batch, dim=dim, dstate=N, seqlen=0, io_dtype=_DTYPE_CODE[io],
                     bc_dtype=_DTYPE_CODE[bc], dt_softplus=int(bool(dt_softplus)),
                     num_chunks=0, flags=flags, reserved=0, workspace=None, workspace_bytes=0)
    rc = library().mamba_selective_state_update(
        _ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(dt_bias), _ptr(out), ctypes.byref(dims), _stream_handle(stream))
    if rc != MAMBA_OK:
        raise MambaError("mamba_selective_state_update", rc)
    return out


def scan_bwd_workspace_bytes(batch, dim, dstate, seqlen, io_dtype=torch.bfloat16,
                             bc_dtype=torch.bfloat16) -> int:
    """Scratch bytes of ``selective_scan_bwd`` on the current device."""
    dims = make_scan_dims(batch, dim, dstate, seqlen, io_dtype, bc_dtype)
    n = library().mamba_selective_scan_bwd_workspace_bytes(ctypes.byref(dims))
    if n == ctypes.c_size_t(-1).value:
        raise MambaError("mamba_selective_scan_bwd_workspace_bytes", -1)
    return int(n)


def selective_scan_bwd(u, delta, A, B, C, dout, D=None, z=None, delta_bias=None, softplus=True,
                       initial_state=None, dlast_state=None, flags=0, workspace=None,
                       stream=None, zoh=False, layout="bdl"):
    """Gradients of the scan through ``mamba_selective_scan_bwd``.

    Same inputs as ``selective_scan_fwd`` plus dout (u's shape and dtype) and
    dlast_state (batch, dim, N) fp32 or None; ``zoh`` sets MAMBA_FLAG_ZOH (the
    zero-order-hold input term, as in the forward) and ``layout="bld"``
    MAMBA_FLAG_LAYOUT_BLD (u, delta, z, dout and their gradients in
    (batch, L, dim)).  Returns a dict: du, ddelta (and dz when z is given) in
    u's shape and dtype; dA, dB, dC (and dD, ddelta_bias, dinitial_state for
    the optional inputs given) in fp32.
    """
    flags, bld = _layout_flags(layout, flags)
    batch, dim, L = _scan_sizes(u, bld)
    act = (batch, L, dim) if bld else (batch, dim, L)
    if zoh:
        flags |= MAMBA_FLAG_ZOH
    N = A.shape[1]
    io, bc = u.dtype, B.dtype
    dev = u.device
    _check_cuda("u", u, (torch.float32, torch.bfloat16), act)
    for name, t in (("delta", delta), ("z", z), ("dout", dout)):
        _check_cuda(name, t, (io,), act)
    _check_cuda("A", A, (torch.float32,), (dim, N))
    _check_cuda("B", B, (torch.float32, torch.bfloat16), (batch, N, L))
    _check_cuda("C", C, (bc,), (batch, N, L))
    _check_cuda("D", D, (torch.float32,), (dim,))
    _check_cuda("delta_bias", delta_bias, (torch.float32,), (dim,))
    _check_cuda("initial_state", initial_state, (torch.float32,), (batch, dim, N))
    _check_cuda("dlast_state", dlast_state, (torch.float32,), (batch, dim, N))
    g = {"du": torch.empty_like(u), "ddelta": torch.empty_like(u),
         "dA": torch.empty((dim, N), dtype=torch.float32, device=dev),
         "dB": torch.empty((batch, N, L), dtype=torch.float32, device=dev),
         "dC": torch.empty((batch, N, L), dtype=torch.float32, device=dev)}
    if z is not None:
        g["dz"] = torch.empty_like(u)
    if D is not None:
        g["dD"] = torch.empty((dim,), dtype=torch.float32, device=dev)
    if delta_bias is not None:
        g["ddelta_bias"] = torch.empty((dim,), dtype=torch.float32, device=dev)
    if initial_state is not None:
        g["dinitial_state"] = torch.empty((batch, dim, N), dtype=torch.float32, device=dev)
    if workspace is None:
        need = scan_bwd_workspace_bytes(batch, dim, N, L, io, bc)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    dims = make_scan_dims(batch, dim, N, L, io, bc, 0, flags, workspace)
    rc = library().mamba_selective_scan_bwd(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        int(bool(softplus)), _ptr(initial_state), _ptr(dout), _ptr(dlast_state), _ptr(g["du"]),
        _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g.get("dD")),
        _ptr(g.get("dz")), _ptr(g.get("ddelta_bias")), _ptr(g.get("dinitial_state")),
        ctypes.byref(dims), _stream_handle(stream))
    if rc != MAMBA_OK:
        raise MambaError("mamba_selective_scan_bwd", rc)
    return g


def _conv_dims(batch, dim, seqlen, io_dtype) -> MambaDims:
    return MambaDims(batch=batch, dim=dim, dstate=1, seqlen=seqlen, io_dtype=_DTYPE_CODE[io_dtype],
                     bc_dtype=_DTYPE_CODE[io_dtype], dt_softplus=0, num_chunks=0, flags=0,
                     reserved=0, workspace=None, workspace_bytes=0)


def causal_conv1d_fwd(x, weight, bias=None, initial_conv_state=None, silu=True, out=None,
                      final_conv_state=None, return_final_state=False, stream=None):
    """Short causal convolution over a sequence through ``mamba_causal_conv1d_fwd``.

    x: (batch, dim, L) fp32 or bf16; weight: (dim, W) fp32, W <= 4; bias: (dim,)
    fp32 or None; initial_conv_state: (batch, dim, W) in x's dtype or None.
    Returns ``out`` (and the final conv state when asked for or given).
    """
    batch, dim, L = x.shape
    W = weight.shape[1]
    io = x.dtype
    _check_cuda("x", x, (torch.float32, torch.bfloat16), (batch, dim, L))
    _check_cuda("weight", weight, (torch.float32,), (dim, W))
    _check_cuda("bias", bias, (torch.float32,), (dim,))
    _check_cuda("initial_conv_state", initial_conv_state, (io,), (batch, dim, W))
    if out is None:
        out = torch.empty_like(x)
    _check_cuda("out", out, (io,), (batch, dim, L))
    if final_conv_state is None and return_final_state:
        final_conv_state = torch.empty((batch, dim, W), dtype=io, device=x.device)
    _check_cuda("final_conv_state", final_conv_state, (io,), (batch, dim, W))
    dims = _conv_dims(batch, dim, L, io)
    rc = library().mamba_causal_conv1d_fwd(
        _ptr(x), _ptr(weight), _ptr(bias), _ptr(initial_conv_state), W, int(bool(silu)),
        _ptr(out), _ptr(final_conv_state), ctypes.byref(dims), _stream_handle(stream))
    if rc != MAMBA_OK:
        raise MambaError("mamba_causal_conv1d_fwd", rc)
    if final_conv_state is not None:
        return out, final_conv_state
    return out


def causal_conv1d_update(conv_state, x, weight, bias=None, silu=True, out=None, stream=None,
                         flags=0):
    """One token of the short convolution through ``mamba_causal_conv1d_update``;
    ``conv_state`` (batch, dim, W) is shifted in place.  ``flags`` may hold
    MAMBA_FLAG_PDL (dependent launch; the previous kernel on the stream must
    not touch this conv state).  Returns ``out`` (batch, dim)."""
    batch, dim, W = conv_state.shape
    io = x.dtype
    _check_cuda("conv_state", conv_state, (io,), (batch, dim, W))
    _check_cuda("x", x, (torch.float32, torch.bfloat16), (batch, dim))
    _check_cuda("weight", weight, (torch.float32,), (dim, W))
    _check_cuda("bias", bias, (torch.float32,), (dim,))
    if out is None:
        out = torch.empty_like(x)
    _check_cuda("out", out, (io,), (batch, dim))
    dims = _conv_dims(batch, dim, 0, io)
    dims.flags = flags
    rc = library().mamba_causal_conv1d_update(
        _ptr(conv_state), _ptr(x), _ptr(weight), _ptr(bias), W, int(bool(silu)), _ptr(out),
        ctypes.byref(dims), _stream_handle(stream))
    if rc != MAMBA_OK:
        raise MambaError("mamba_causal_conv1d_update", rc)
    return out


def ssd_chunk_scan_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True,
                       initial_state=None, out=None, final_state=None,
                       return_final_state=False, stream=None):
    """Mamba-2 layer (scalar A per head) through ``mamba_ssd_chunk_scan_fwd``.

    x, z: (batch, L, nheads, 64) bf16; dt: (batch, L, nheads) bf16; A, D,
    dt_bias: (nheads,) fp32; B, C: (batch, L, ngroups, 128) bf16;
    initial_state: (batch, nheads, 64, 128) fp32 or None.  Returns out (like
    x), or (out, final_state) when ``return_final_state`` is set or a
    ``final_state`` buffer is passed.  Delta must be non-negative (softplus on,
    or dt + dt_bias >= 0 with it off).
    """
    batch, L, nheads, headdim = x.shape
    ngroups, dstate = B.shape[2], B.shape[3]
    bf = (torch.bfloat16,)
    _check_cuda("x", x, bf, (batch, L, nheads, headdim))
    _check_cuda("dt", dt, bf, (batch, L, nheads))
    _check_cuda("A", A, (torch.float32,), (nheads,))
    _check_cuda("B", B, bf, (batch, L, ngroups, dstate))
    _check_cuda("C", C, bf, (batch, L, ngroups, dstate))
    _check_cuda("D", D, (torch.float32,), (nheads,))
    _check_cuda("z", z, bf, (batch, L, nheads, headdim))
    _check_cuda("dt_bias", dt_bias, (torch.float32,), (nheads,))
    st_shape = (batch, nheads, headdim, dstate)
    _check_cuda("initial_state", initial_state, (torch.float32,), st_shape)
    if out is None:
        out = torch.empty_like(x)
    _check_cuda("out", out, bf, tuple(x.shape))
    if final_state is None and return_final_state:
        final_state = torch.empty(st_shape, dtype=torch.float32, device=x.device)
    _check_cuda("final_state", final_state, (torch.float32,), st_shape)
    dims = SsdDims(batch=batch, seqlen=L, nheads=nheads, headdim=headdim, ngroups=ngroups,
                   dstate=dstate, io_dtype=MAMBA_BF16, dt_softplus=int(bool(dt_softplus)))
    rc = library().mamba_ssd_chunk_scan_fwd(
        _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
        _ptr(initial_state), _ptr(out), _ptr(final_state), ctypes.byref(dims),
        _stream_handle(stream))
    if rc != MAMBA_OK:
        raise MambaError("mamba_ssd_chunk_scan_fwd", rc)
    if return_final_state or final_state is not None:
        return out, final_state
    return out


def device_status() -> int:
    """Read and clear the library's device-side status word (synchronises)."""
    return int(library().mamba_device_status())
