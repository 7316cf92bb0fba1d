"""Float64 CPU oracle: ctypes wrapper around ``ssm_oracle.c``.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm are the only callers.  The CUDA
library never imports, links or runs anything here, and nothing here imports
the CUDA library.

What it computes (float64, plain sequential recurrence):

    Delta_t  = softplus(delta_t + bias_d)            (softplus may be off)
    h_t,n    = exp(Delta_t * A_d,n) * h_{t-1},n + Delta_t * B_t,n * u_t
    y_t      = sum_n C_t,n * h_t,n + D_d * u_t
    out_t    = y_t * silu(z_t)                       (z optional)

from h_{-1} = 0, or from a given ``initial_state``.  With ``zoh=True`` the input
term is the zero-order-hold one, expm1(Delta_t A_d,n) / A_d,n * B_t,n * u_t
(Delta_t B_t,n u_t where A_d,n = 0), i.e. Bbar = (Delta A)^-1 (exp(Delta A) - I)
Delta B for the diagonal A.

The backward pass of the scan (Euler or zero-order-hold input term) is the
adjoint recurrence in reverse time; ``selective_scan_bwd`` returns the
gradients of a linear functional of out and last_state.

``ssd_scan`` is the Mamba-2 layer ("Mamba 与状态空间模型", section
"Mamba-2：两种算法"): A is a scalar per head, the state of a head is a
(headdim x dstate) matrix, B and C are shared by the heads of a group, and the
recurrence S_t = exp(Delta_t A_h) S_{t-1} + Delta_t x_t B_t^T, y_t = S_t C_t
+ D_h x_t is run one step at a time.

The block's short causal convolution (depthwise, W taps, optional silu) and
its single-token update are the plain weighted sums over the window ("Mamba 与
状态空间模型", section 固定大小的状态: a short convolution keeps the 4 most
recent inputs of each channel).

Following "超越注意力：探索Mamba与状态空间模型" (sections 状态空间模型基础 for
the zero-order hold, 选择性状态空间模型, 代码实现概览 for the Euler default) and
"Mamba 与状态空间模型" (section 由词元决定).  The update is the same single step
applied to a given state.

Every input is converted to contiguous float64 first; bf16 and fp32 values
convert exactly, so the oracle sees the same numbers the GPU sees.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SOURCE = HERE / "ssm_oracle.c"
BUILD_DIR = HERE / "_build"
LIBRARY = BUILD_DIR / "libssm_oracle.so"


def build(source: Path = SOURCE, output: Path = LIBRARY, force: bool = False) -> Path:
    """Compile the C oracle with gcc (-O2, OpenMP, no fast-math)."""
    source, output = Path(source), Path(output)
    if not force and output.exists() and output.stat().st_mtime >= source.stat().st_mtime:
        return output
    output.parent.mkdir(parents=True, exist_ok=True)
    tmp = output.with_suffix(f".{os.getpid()}.tmp.so")
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
           str(source), "-o", str(tmp), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, output)
    return output


def _f64(a):
    """Contiguous float64 numpy copy of an array-like (numpy or CPU torch)."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


class Oracle:
    """Handle on one compiled oracle library (the default one, or a test build)."""

    def __init__(self, library: Path | str | None = None):
        path = Path(library) if library is not None else build()
        self.path = path
        self._lib = ctypes.CDLL(str(path))
        dp = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        ci = ctypes.c_int
        self._lib.oracle_selective_scan_ex_f64.restype = ctypes.c_int
        self._lib.oracle_selective_scan_ex_f64.argtypes = [
            i64, i64, i64, i64, dp, dp, dp, dp, dp, dp, dp, dp, ci, ci, dp, dp, dp]
        self._lib.oracle_selective_state_update_ex_f64.restype = ctypes.c_int
        self._lib.oracle_selective_state_update_ex_f64.argtypes = [
            i64, i64, i64, dp, dp, dp, dp, dp, dp, dp, dp, dp, ci, ci, dp, dp]
        self._lib.oracle_selective_scan_bwd_ex_f64.restype = ctypes.c_int
        self._lib.oracle_selective_scan_bwd_ex_f64.argtypes = [
            i64, i64, i64, i64, dp, dp, dp, dp, dp, dp, dp, dp, ci, ci, dp, dp, dp,
            dp, dp, dp, dp, dp, dp, dp, dp, dp]
        self._lib.oracle_causal_conv1d_f64.restype = ctypes.c_int
        self._lib.oracle_causal_conv1d_f64.argtypes = [
            i64, i64, i64, i64, dp, dp, dp, dp, ci, dp, dp]
        self._lib.oracle_causal_conv1d_update_f64.restype = ctypes.c_int
        self._lib.oracle_causal_conv1d_update_f64.argtypes = [
            i64, i64, i64, dp, dp, dp, dp, ci, dp, dp]
        self._lib.oracle_ssd_scan_f64.restype = ctypes.c_int
        self._lib.oracle_ssd_scan_f64.argtypes = [
            i64, i64, i64, i64, i64, i64, dp, dp, dp, dp, dp, dp, dp, dp, ci, dp, dp, dp]
        self._lib.oracle_num_threads.restype = ctypes.c_int
        self._lib.oracle_num_threads.argtypes = []
        self._lib.oracle_set_num_threads.restype = None
        self._lib.oracle_set_num_threads.argtypes = [ctypes.c_int]

    def num_threads(self) -> int:
        return int(self._lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        """Threads of the oracle's later parallel loops (timing only; results
        do not depend on it)."""
        self._lib.oracle_set_num_threads(int(n))

    def selective_scan(self, u, delta, A, B, C, D=None, z=None, delta_bias=None,
                       softplus=True, zoh=False, initial_state=None):
        """Return (out, last_state) as float64 arrays.

        u, delta, z: (batch, dim, L); B, C: (batch, N, L); A: (dim, N);
        D, delta_bias: (dim,); initial_state: (batch, dim, N) or None (zeros).
        out: (batch, dim, L); last_state: (batch, dim, N).
        """
        u, delta, A, B, C = map(_f64, (u, delta, A, B, C))
        D, z, delta_bias, initial_state = map(_f64, (D, z, delta_bias, initial_state))
        batch, dim, seqlen = u.shape
        dstate = A.shape[1]
        assert delta.shape == u.shape and A.shape == (dim, dstate)
        assert B.shape == (batch, dstate, seqlen) and C.shape == B.shape
        assert z is None or z.shape == u.shape
        assert D is None or D.shape == (dim,)
        assert delta_bias is None or delta_bias.shape == (dim,)
        assert initial_state is None or initial_state.shape == (batch, dim, dstate)
        out = np.empty_like(u)
        last_state = np.empty((batch, dim, dstate), dtype=np.float64)
        rc = self._lib.oracle_selective_scan_ex_f64(
            batch, dim, dstate, seqlen, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
            _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(softplus)), int(bool(zoh)),
            _ptr(initial_state), _ptr(out), _ptr(last_state))
        if rc != 0:
            raise ValueError(f"oracle_selective_scan_f64 returned {rc}")
        return out, last_state

    def selective_state_update(self, state, x, dt, A, B, C, D=None, z=None, dt_bias=None,
                               dt_softplus=True, zoh=False):
        """Return (new_state, out) as float64 arrays; the input state is not modified.
        ``zoh`` selects the zero-order-hold input term, as in ``selective_scan``.

        state: (batch, dim, N); x, dt, z: (batch, dim); B, C: (batch, N);
        A: (dim, N); D, dt_bias: (dim,).
        """
        state, x, dt, A, B, C = map(_f64, (state, x, dt, A, B, C))
        D, z, dt_bias = map(_f64, (D, z, dt_bias))
        batch, dim, dstate = state.shape
        assert x.shape == (batch, dim) and dt.shape == x.shape
        assert A.shape == (dim, dstate) and B.shape == (batch, dstate) and C.shape == B.shape
        assert z is None or z.shape == x.shape
        new_state = np.empty_like(state)
        out = np.empty_like(x)
        rc = self._lib.oracle_selective_state_update_ex_f64(
            batch, dim, dstate, _ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
            _ptr(D), _ptr(z), _ptr(dt_bias), int(bool(dt_softplus)), int(bool(zoh)),
            _ptr(new_state), _ptr(out))
        if rc != 0:
            raise ValueError(f"oracle_selective_state_update_f64 returned {rc}")
        return new_state, out

    def selective_scan_bwd(self, u, delta, A, B, C, dout, D=None, z=None, delta_bias=None,
                           softplus=True, initial_state=None, dlast_state=None, zoh=False):
        """Gradients of sum(dout * out) + sum(dlast_state * last_state) of the
        scan (Euler input term, or zero-order hold with ``zoh``), as a dict of
        float64 arrays: du, ddelta, dA, dB, dC, and dD, dz, ddelta_bias,
        dinitial_state for the optional inputs given."""
        u, delta, A, B, C, dout = map(_f64, (u, delta, A, B, C, dout))
        D, z, delta_bias = map(_f64, (D, z, delta_bias))
        initial_state, dlast_state = _f64(initial_state), _f64(dlast_state)
        batch, dim, seqlen = u.shape
        dstate = A.shape[1]
        assert dout.shape == u.shape and delta.shape == u.shape
        assert B.shape == (batch, dstate, seqlen) and C.shape == B.shape
        g = {"du": np.empty_like(u), "ddelta": np.empty_like(u), "dA": np.empty_like(A),
             "dB": np.empty_like(B), "dC": np.empty_like(C)}
        if D is not None:
            g["dD"] = np.empty_like(D)
        if z is not None:
            g["dz"] = np.empty_like(z)
        if delta_bias is not None:
            g["ddelta_bias"] = np.empty_like(delta_bias)
        if initial_state is not None:
            g["dinitial_state"] = np.empty_like(initial_state)
        rc = self._lib.oracle_selective_scan_bwd_ex_f64(
            batch, dim, dstate, seqlen, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
            _ptr(z), _ptr(delta_bias), int(bool(softplus)), int(bool(zoh)), _ptr(initial_state),
            _ptr(dout),
            _ptr(dlast_state), _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]),
            _ptr(g["dC"]), _ptr(g.get("dD")), _ptr(g.get("dz")), _ptr(g.get("ddelta_bias")),
            _ptr(g.get("dinitial_state")))
        if rc != 0:
            raise ValueError(f"oracle_selective_scan_bwd_ex_f64 returned {rc}")
        return g

    def causal_conv1d(self, x, weight, bias=None, initial_conv_state=None, silu=True):
        """Return (out, final_conv_state) as float64 arrays.

        x: (batch, dim, L); weight: (dim, W); bias: (dim,); initial_conv_state:
        (batch, dim, W), the W inputs before t = 0, oldest first (None: zeros).
        final_conv_state: (batch, dim, W), the last W inputs.
        """
        x, weight = _f64(x), _f64(weight)
        bias, init = _f64(bias), _f64(initial_conv_state)
        batch, dim, seqlen = x.shape
        width = weight.shape[1]
        assert weight.shape == (dim, width)
        assert bias is None or bias.shape == (dim,)
        assert init is None or init.shape == (batch, dim, width)
        out = np.empty_like(x)
        final = np.empty((batch, dim, width), dtype=np.float64)
        rc = self._lib.oracle_causal_conv1d_f64(batch, dim, seqlen, width, _ptr(x), _ptr(weight),
                                                _ptr(bias), _ptr(init), int(bool(silu)),
                                                _ptr(out), _ptr(final))
        if rc != 0:
            raise ValueError(f"oracle_causal_conv1d_f64 returned {rc}")
        return out, final

    def causal_conv1d_update(self, conv_state, x, weight, bias=None, silu=True):
        """Return (new_conv_state, out) as float64 arrays; conv_state: (batch, dim, W)
        is not modified; x: (batch, dim)."""
        conv_state, x, weight, bias = _f64(conv_state), _f64(x), _f64(weight), _f64(bias)
        batch, dim, width = conv_state.shape
        assert x.shape == (batch, dim) and weight.shape == (dim, width)
        new = np.empty_like(conv_state)
        out = np.empty_like(x)
        rc = self._lib.oracle_causal_conv1d_update_f64(batch, dim, width, _ptr(conv_state), _ptr(x),
                                                       _ptr(weight), _ptr(bias), int(bool(silu)),
                                                       _ptr(new), _ptr(out))
        if rc != 0:
            raise ValueError(f"oracle_causal_conv1d_update_f64 returned {rc}")
        return new, out

    def ssd_scan(self, x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True,
                 initial_state=None):
        """Mamba-2 layer with a scalar A per head, as the plain recurrence.

        x, z: (batch, L, nheads, headdim); dt: (batch, L, nheads); A, D, dt_bias:
        (nheads,); B, C: (batch, L, ngroups, dstate); initial_state: (batch,
        nheads, headdim, dstate).  Returns (out, final_state) as float64 arrays,
        out shaped like x and final_state (batch, nheads, headdim, dstate).
        """
        x, dt, A, B, C = map(_f64, (x, dt, A, B, C))
        D, z, dt_bias, init = map(_f64, (D, z, dt_bias, initial_state))
        batch, seqlen, nheads, headdim = x.shape
        ngroups, dstate = B.shape[2], B.shape[3]
        assert dt.shape == (batch, seqlen, nheads) and A.shape == (nheads,)
        assert B.shape == (batch, seqlen, ngroups, dstate) and C.shape == B.shape
        assert z is None or z.shape == x.shape
        assert init is None or init.shape == (batch, nheads, headdim, dstate)
        out = np.empty_like(x)
        final = np.empty((batch, nheads, headdim, dstate), dtype=np.float64)
        rc = self._lib.oracle_ssd_scan_f64(batch, seqlen, nheads, headdim, ngroups, dstate,
                                           _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                           _ptr(z), _ptr(dt_bias), int(bool(dt_softplus)),
                                           _ptr(init), _ptr(out), _ptr(final))
        if rc != 0:
            raise ValueError(f"oracle_ssd_scan_f64 returned {rc}")
        return out, final


_DEFAULT: Oracle | None = None


def default() -> Oracle:
    """The oracle built from ``ssm_oracle.c`` (compiled on first use)."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT
