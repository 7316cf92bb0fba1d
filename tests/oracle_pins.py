"""Pins for the float64 oracle: checks against what the pages and mathematics fix.

Each pin takes an ``oracle.oracle.Oracle`` handle and raises AssertionError when
the handle disagrees with an independent statement of the result.  None of
them re-evaluates the oracle's recurrence: they use the unrolled sum, the LTI
convolution, the gated-RNN form, the limits of Delta, closed values and
invariants.  The mutation test runs every pin against deliberately broken
copies of the oracle to show that a plausible slip is caught by at least one.

Sources (page title, section):
  - "超越注意力：探索Mamba与状态空间模型", 状态空间模型基础: discretisation and
    the recurrence; the LTI system is a convolution.
  - "Mamba 与状态空间模型", 每一步都一样: a time-invariant SSM is a convolution
    with a fixed kernel; A is initialised to -1 ... -16.
  - same page, 由词元决定: large Delta resets the state to the current input,
    small Delta holds it; with a one-number state the update is the gate
    h <- (1 - g) h + g x (Theorem 1).
  - "超越注意力：探索Mamba与状态空间模型", 状态空间模型基础: the zero-order-hold
    input matrix Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B.  Under it the
    Theorem-1 gate holds with B = 1 and no rescaling, and a constant input has
    the fixed point h* = -B u / A for every Delta.
  - "Mamba 与状态空间模型", Mamba-2：两种算法: with A a scalar per head the layer
    is a lower-triangular matrix (C at step i, B at step j, the decay between);
    a sequence can be cut into pieces that pass only the state on.
"""
from __future__ import annotations

import math

import numpy as np


def _rel(got, want):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    scale = max(float(np.max(np.abs(want))) if want.size else 0.0, 1e-300)
    return float(np.max(np.abs(got - want))) / scale if want.size else 0.0


def _close(got, want, tol, what):
    err = _rel(got, want)
    assert err <= tol, f"{what}: relative error {err:.3e} > {tol:.1e}"


def _random_problem(seed, batch=2, dim=3, dstate=4, seqlen=40):
    rng = np.random.default_rng(seed)
    return dict(
        u=rng.standard_normal((batch, dim, seqlen)),
        delta=rng.uniform(0.05, 0.6, (batch, dim, seqlen)),
        A=-rng.uniform(0.2, 2.0, (dim, dstate)),
        B=rng.standard_normal((batch, dstate, seqlen)),
        C=rng.standard_normal((batch, dstate, seqlen)),
        D=rng.standard_normal(dim),
        delta_bias=rng.uniform(0.0, 0.1, dim),
    )


def pin_unrolled_sum(o):
    """y_t = sum_{s<=t} C_t (prod_{s<r<=t} Abar_r) Delta_s B_s u_s + D u_t, brute force.

    Softplus off so Delta = delta + bias is fixed by the inputs alone.  Also
    checks last_state = the same sum at t = L-1 without the C_t factor.
    """
    p = _random_problem(11)
    out, last = o.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                 delta_bias=p["delta_bias"], softplus=False)
    u, A, B, C, D = p["u"], p["A"], p["B"], p["C"], p["D"]
    Delta = p["delta"] + p["delta_bias"][None, :, None]
    batch, dim, L = u.shape
    want = np.zeros_like(u)
    want_last = np.zeros((batch, dim, A.shape[1]))
    for b in range(batch):
        for d in range(dim):
            abar = np.exp(Delta[b, d][:, None] * A[d][None, :])        # (L, N)
            for t in range(L):
                acc = 0.0
                for s in range(t + 1):
                    decay = np.prod(abar[s + 1:t + 1], axis=0)          # (N,)
                    acc += np.sum(C[b, :, t] * decay * Delta[b, d, s] * B[b, :, s]) * u[b, d, s]
                want[b, d, t] = acc + D[d] * u[b, d, t]
            for s in range(L):
                decay = np.prod(abar[s + 1:L], axis=0)
                want_last[b, d] += decay * Delta[b, d, s] * B[b, :, s] * u[b, d, s]
    _close(out, want, 1e-12, "unrolled sum: out")
    _close(last, want_last, 1e-12, "unrolled sum: last_state")


def pin_gate_closed_values(o):
    """out = y * silu(z) with silu at closed values: silu(0)=0, silu(+-ln 3)=(3/4)ln 3,
    -(1/4)ln 3, silu(40) = 40 to 1e-16."""
    p = _random_problem(12, batch=1, dim=2, seqlen=8)
    y, _ = o.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                            delta_bias=p["delta_bias"], softplus=True)
    ln3 = math.log(3.0)
    zvals = np.array([0.0, ln3, -ln3, 40.0, 0.0, ln3, -ln3, 40.0])
    silu = np.array([0.0, 0.75 * ln3, -0.25 * ln3, 40.0, 0.0, 0.75 * ln3, -0.25 * ln3, 40.0])
    z = np.broadcast_to(zvals, p["u"].shape).copy()
    out, _ = o.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=z,
                              delta_bias=p["delta_bias"], softplus=True)
    _close(out, y * silu[None, None, :], 1e-14, "gate closed values")


def pin_lti_convolution(o):
    """Delta, B, C constant in t: y = u * K + D u with K_k = sum_n C_n Abar_n^k Delta B_n."""
    rng = np.random.default_rng(13)
    batch, dim, N, L = 2, 3, 4, 48
    u = rng.standard_normal((batch, dim, L))
    Dl = rng.uniform(0.05, 0.5, (batch, dim))
    delta = np.broadcast_to(Dl[:, :, None], (batch, dim, L)).copy()
    A = -rng.uniform(0.1, 1.5, (dim, N))
    Bc = rng.standard_normal((batch, N))
    Cc = rng.standard_normal((batch, N))
    B = np.broadcast_to(Bc[:, :, None], (batch, N, L)).copy()
    C = np.broadcast_to(Cc[:, :, None], (batch, N, L)).copy()
    D = rng.standard_normal(dim)
    out, _ = o.selective_scan(u, delta, A, B, C, D=D, softplus=False)
    want = np.zeros_like(u)
    k = np.arange(L)
    for b in range(batch):
        for d in range(dim):
            abar = np.exp(Dl[b, d] * A[d])                                   # (N,)
            K = np.sum(Cc[b][None, :] * np.power(abar[None, :], k[:, None])
                       * Dl[b, d] * Bc[b][None, :], axis=1)                  # (L,)
            want[b, d] = np.convolve(u[b, d], K)[:L] + D[d] * u[b, d]
    _close(out, want, 1e-12, "LTI convolution")


def pin_gated_rnn_theorem1(o):
    """N=1, A=-1, softplus on, C=1: with B_t = g_t / Delta_t the scan is the gate
    h_t = (1-g_t) h_{t-1} + g_t x_t, g = sigmoid(delta + bias), since
    1 - exp(-softplus(s)) = sigmoid(s)."""
    rng = np.random.default_rng(14)
    batch, L = 3, 64
    s_delta = rng.standard_normal((batch, 1, L)) * 2.0
    bias = np.array([-0.7])
    s = s_delta + bias[None, :, None]
    g = 1.0 / (1.0 + np.exp(-s))
    Delta = np.log1p(np.exp(s))
    x = rng.standard_normal((batch, 1, L))
    B = (g / Delta).reshape(batch, 1, L)
    C = np.ones((batch, 1, L))
    A = np.array([[-1.0]])
    out, last = o.selective_scan(x, s_delta, A, B, C, delta_bias=bias, softplus=True)
    want = np.zeros_like(x)
    for b in range(batch):
        h = 0.0
        for t in range(L):
            h = (1.0 - g[b, 0, t]) * h + g[b, 0, t] * x[b, 0, t]
            want[b, 0, t] = h
    _close(out, want, 1e-12, "gated RNN (Theorem 1)")
    _close(last[:, :, 0], want[:, :, -1], 1e-12, "gated RNN last state")


def pin_small_delta_holds(o):
    """Delta -> 0 holds the state: write once with Delta = softplus(40), then Delta ~ e^-80."""
    rng = np.random.default_rng(15)
    batch, dim, N, L = 1, 2, 4, 32
    u = rng.standard_normal((batch, dim, L))
    delta = np.full((batch, dim, L), -80.0)
    delta[:, :, 0] = 40.0
    A = -np.tile(np.arange(1, N + 1, dtype=np.float64), (dim, 1))
    B = rng.standard_normal((batch, N, L))
    C = rng.standard_normal((batch, N, L))
    D = rng.standard_normal(dim)
    out, last = o.selective_scan(u, delta, A, B, C, D=D, softplus=True)
    h0 = 40.0 * B[:, None, :, 0] * u[:, :, 0][:, :, None]                  # (b, d, N)
    want = np.einsum("bdn,bnt->bdt", h0, C) + D[None, :, None] * u
    _close(out, want, 1e-12, "small Delta holds the state")
    _close(last, h0, 1e-12, "small Delta: last_state")


def pin_large_delta_resets(o):
    """Large Delta with A <= -1: Abar underflows to 0, h_t = Delta B_t u_t (no history)."""
    rng = np.random.default_rng(16)
    batch, dim, N, L = 2, 3, 4, 20
    u = rng.standard_normal((batch, dim, L))
    delta = np.full((batch, dim, L), 1000.0)
    A = -rng.uniform(1.0, 3.0, (dim, N))
    B = rng.standard_normal((batch, N, L))
    C = rng.standard_normal((batch, N, L))
    D = rng.standard_normal(dim)
    out, last = o.selective_scan(u, delta, A, B, C, D=D, softplus=False)
    want = 1000.0 * np.einsum("bnt,bnt->bt", C, B)[:, None, :] * u + D[None, :, None] * u
    _close(out, want, 1e-13, "large Delta resets the state")
    _close(last, 1000.0 * B[:, None, :, -1] * u[:, :, -1][:, :, None], 1e-13,
           "large Delta: last_state")


def pin_zero_A_cumulative_sum(o):
    """A = 0 gives Abar = 1: h_t = cumulative sum of Delta_s B_s u_s."""
    p = _random_problem(17, seqlen=33)
    A = np.zeros_like(p["A"])
    out, last = o.selective_scan(p["u"], p["delta"], A, p["B"], p["C"], D=p["D"],
                                 delta_bias=p["delta_bias"], softplus=False)
    Delta = p["delta"] + p["delta_bias"][None, :, None]
    inc = Delta[:, :, None, :] * p["B"][:, None, :, :] * p["u"][:, :, None, :]   # b d n t
    h = np.cumsum(inc, axis=-1)
    want = np.einsum("bdnt,bnt->bdt", h, p["C"]) + p["D"][None, :, None] * p["u"]
    _close(out, want, 1e-12, "A = 0 cumulative sum")
    _close(last, h[..., -1], 1e-12, "A = 0 last_state")


def pin_softplus_closed_values(o):
    """With N=1, A=0, B=C=u=1, L=1 the output is Delta itself:
    softplus(0) = ln 2, softplus(ln(e-1)) = 1, softplus(log(expm1(v))) = v,
    softplus(50) = 50, softplus(-50) = e^-50 (to 1e-21 relative)."""
    v = 0.037
    s = np.array([0.0, math.log(math.e - 1.0), math.log(math.expm1(v)), 50.0, -50.0])
    want = np.array([math.log(2.0), 1.0, v, 50.0, math.exp(-50.0)])
    dim = s.size
    ones = np.ones((1, dim, 1))
    out, _ = o.selective_scan(ones, s.reshape(1, dim, 1), np.zeros((dim, 1)),
                              np.ones((1, 1, 1)), np.ones((1, 1, 1)), softplus=True)
    got = out.reshape(-1)
    err = np.abs(got - want) / np.abs(want)
    assert np.all(err <= 1e-14), f"softplus closed values: {got} vs {want}"
    # split between delta and delta_bias: the bias is added before softplus
    out2, _ = o.selective_scan(ones, (s - 0.25).reshape(1, dim, 1), np.zeros((dim, 1)),
                               np.ones((1, 1, 1)), np.ones((1, 1, 1)),
                               delta_bias=np.full(dim, 0.25), softplus=True)
    _close(out2.reshape(-1), want, 1e-14, "softplus with bias")


def pin_linearity_and_causality(o):
    """Without the gate, out is linear in u (B, C, Delta fixed) and causal."""
    p = _random_problem(18, seqlen=30)
    rng = np.random.default_rng(19)
    u2 = rng.standard_normal(p["u"].shape)
    args = (p["A"], p["B"], p["C"])
    kw = dict(D=p["D"], delta_bias=p["delta_bias"], softplus=True)
    y1, _ = o.selective_scan(p["u"], p["delta"], *args, **kw)
    y2, _ = o.selective_scan(u2, p["delta"], *args, **kw)
    y12, _ = o.selective_scan(2.5 * p["u"] - 0.75 * u2, p["delta"], *args, **kw)
    _close(y12, 2.5 * y1 - 0.75 * y2, 1e-12, "linearity in u")
    s0 = 17
    u3 = p["u"].copy()
    u3[:, :, s0] += 1.0
    y3, _ = o.selective_scan(u3, p["delta"], *args, **kw)
    assert np.array_equal(y3[:, :, :s0], y1[:, :, :s0]), "causality: earlier outputs moved"
    assert np.all(np.abs(y3[:, :, s0] - y1[:, :, s0]) > 0), "perturbation had no effect"


def _decode_problem(seed, batch=2, dim=3, N=4, T=24):
    rng = np.random.default_rng(seed)
    return dict(
        x=rng.standard_normal((batch, dim, T)),
        dt=rng.standard_normal((batch, dim, T)),
        z=rng.standard_normal((batch, dim, T)),
        A=-rng.uniform(0.2, 2.0, (dim, N)),
        B=rng.standard_normal((batch, N, T)) / 4,
        C=rng.standard_normal((batch, N, T)) / 4,
        D=rng.standard_normal(dim),
        bias=rng.uniform(-1.0, 0.0, dim),
    )


def pin_update_steps_equal_scan(o):
    """T single-token updates from the zero state reproduce the scan over the same T tokens."""
    p = _decode_problem(21)
    out_scan, last = o.selective_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], D=p["D"],
                                      z=p["z"], delta_bias=p["bias"], softplus=True)
    batch, dim, T = p["x"].shape
    state = np.zeros((batch, dim, p["A"].shape[1]))
    outs = np.zeros_like(p["x"])
    for t in range(T):
        state, outs[:, :, t] = o.selective_state_update(
            state, p["x"][:, :, t], p["dt"][:, :, t], p["A"], p["B"][:, :, t],
            p["C"][:, :, t], D=p["D"], z=p["z"][:, :, t], dt_bias=p["bias"], dt_softplus=True)
    _close(outs, out_scan, 1e-13, "update steps = scan: out")
    _close(state, last, 1e-13, "update steps = scan: state")


def pin_update_continues_scan(o):
    """Updates started from the scan's last_state after T1 tokens continue it exactly."""
    p = _decode_problem(22, T=30)
    T1 = 18
    out_full, last_full = o.selective_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], D=p["D"],
                                           z=p["z"], delta_bias=p["bias"], softplus=True)
    _, state = o.selective_scan(p["x"][:, :, :T1], p["dt"][:, :, :T1], p["A"],
                                p["B"][:, :, :T1], p["C"][:, :, :T1], D=p["D"],
                                z=p["z"][:, :, :T1], delta_bias=p["bias"], softplus=True)
    outs = []
    for t in range(T1, p["x"].shape[2]):
        state, y = o.selective_state_update(
            state, p["x"][:, :, t], p["dt"][:, :, t], p["A"], p["B"][:, :, t],
            p["C"][:, :, t], D=p["D"], z=p["z"][:, :, t], dt_bias=p["bias"], dt_softplus=True)
        outs.append(y)
    _close(np.stack(outs, axis=-1), out_full[:, :, T1:], 1e-13, "update continues scan: out")
    _close(state, last_full, 1e-13, "update continues scan: state")


def pin_update_limits(o):
    """Update with large Delta resets the state to Delta B x; with tiny Delta it holds it."""
    rng = np.random.default_rng(23)
    batch, dim, N = 2, 3, 4
    state = rng.standard_normal((batch, dim, N))
    x = rng.standard_normal((batch, dim))
    A = -rng.uniform(1.0, 2.0, (dim, N))
    B = rng.standard_normal((batch, N))
    C = rng.standard_normal((batch, N))
    D = rng.standard_normal(dim)
    new, out = o.selective_state_update(state, x, np.full((batch, dim), 1000.0), A, B, C,
                                        D=D, dt_softplus=False)
    reset = 1000.0 * B[:, None, :] * x[:, :, None]
    _close(new, reset, 1e-13, "update reset: state")
    _close(out, np.einsum("bdn,bn->bd", reset, C) + D[None, :] * x, 1e-13, "update reset: out")
    new, out = o.selective_state_update(state, x, np.full((batch, dim), -80.0), A, B, C,
                                        D=D, dt_softplus=True)
    _close(new, state, 1e-13, "update hold: state")
    _close(out, np.einsum("bdn,bn->bd", state, C) + D[None, :] * x, 1e-13, "update hold: out")


def pin_zoh_gated_rnn_exact(o):
    """Zero-order hold, N=1, A=-1, B=C=1, softplus on: Bbar = 1 - exp(-Delta) = g with
    g = sigmoid(delta + bias), so the scan is exactly h_t = (1-g_t) h_{t-1} + g_t x_t."""
    rng = np.random.default_rng(31)
    batch, L = 2, 64
    s_delta = rng.standard_normal((batch, 1, L)) * 2.0
    bias = np.array([0.3])
    g = 1.0 / (1.0 + np.exp(-(s_delta + bias[None, :, None])))
    x = rng.standard_normal((batch, 1, L))
    ones = np.ones((batch, 1, L))
    out, last = o.selective_scan(x, s_delta, np.array([[-1.0]]), ones, ones, delta_bias=bias,
                                 softplus=True, zoh=True)
    want = np.zeros_like(x)
    for b in range(batch):
        h = 0.0
        for t in range(L):
            h = (1.0 - g[b, 0, t]) * h + g[b, 0, t] * x[b, 0, t]
            want[b, 0, t] = h
    _close(out, want, 1e-12, "zero-order hold gate (Theorem 1)")
    _close(last[:, :, 0], want[:, :, -1], 1e-12, "zero-order hold gate: last state")


def pin_zoh_fixed_point(o):
    """Zero-order hold with u and B constant in time: h* = -B u / A is a fixed point for
    any Delta sequence, so starting there the state never moves and y_t = C_t h* + D u."""
    rng = np.random.default_rng(32)
    batch, dim, N, L = 2, 3, 4, 40
    A = -rng.uniform(0.2, 2.0, (dim, N))
    ubd = rng.standard_normal((batch, dim))
    Bbn = rng.standard_normal((batch, N))
    u = np.broadcast_to(ubd[:, :, None], (batch, dim, L)).copy()
    B = np.broadcast_to(Bbn[:, :, None], (batch, N, L)).copy()
    C = rng.standard_normal((batch, N, L))
    D = rng.standard_normal(dim)
    delta = rng.uniform(0.01, 2.0, (batch, dim, L))
    h_star = -Bbn[:, None, :] * ubd[:, :, None] / A[None, :, :]          # (b, d, N)
    out, last = o.selective_scan(u, delta, A, B, C, D=D, softplus=False, zoh=True,
                                 initial_state=h_star)
    want = np.einsum("bdn,bnt->bdt", h_star, C) + D[None, :, None] * u
    _close(out, want, 1e-12, "zero-order hold fixed point: out")
    _close(last, h_star, 1e-12, "zero-order hold fixed point: last_state")


def pin_zoh_zero_A_is_cumulative_sum(o):
    """Zero-order hold at A = 0: the gain's limit is Delta, so h_t = sum_s Delta_s B_s u_s."""
    p = _random_problem(33, seqlen=29)
    A = np.zeros_like(p["A"])
    out, last = o.selective_scan(p["u"], p["delta"], A, p["B"], p["C"], D=p["D"],
                                 delta_bias=p["delta_bias"], softplus=False, zoh=True)
    Delta = p["delta"] + p["delta_bias"][None, :, None]
    h = np.cumsum(Delta[:, :, None, :] * p["B"][:, None, :, :] * p["u"][:, :, None, :], axis=-1)
    want = np.einsum("bdnt,bnt->bdt", h, p["C"]) + p["D"][None, :, None] * p["u"]
    _close(out, want, 1e-12, "zero-order hold, A = 0: out")
    _close(last, h[..., -1], 1e-12, "zero-order hold, A = 0: last_state")


def pin_zoh_unrolled_sum(o):
    """Zero-order hold, brute force: y_t = sum_{s<=t} C_t (prod_{s<r<=t} Abar_r)
    (Abar_s - 1) / A B_s u_s + D u_t."""
    p = _random_problem(34, seqlen=24)
    out, last = o.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                 delta_bias=p["delta_bias"], softplus=False, zoh=True)
    u, A, B, C, D = p["u"], p["A"], p["B"], p["C"], p["D"]
    Delta = p["delta"] + p["delta_bias"][None, :, None]
    batch, dim, L = u.shape
    want = np.zeros_like(u)
    want_last = np.zeros((batch, dim, A.shape[1]))
    for b in range(batch):
        for d in range(dim):
            abar = np.exp(Delta[b, d][:, None] * A[d][None, :])        # (L, N)
            bbar = (abar - 1.0) / A[d][None, :]                          # (L, N) per unit B
            for t in range(L):
                acc = 0.0
                for s in range(t + 1):
                    decay = np.prod(abar[s + 1:t + 1], axis=0)
                    acc += np.sum(C[b, :, t] * decay * bbar[s] * B[b, :, s]) * u[b, d, s]
                want[b, d, t] = acc + D[d] * u[b, d, t]
            for s in range(L):
                want_last[b, d] += np.prod(abar[s + 1:L], axis=0) * bbar[s] * B[b, :, s] * u[b, d, s]
    _close(out, want, 1e-11, "zero-order hold unrolled sum: out")
    _close(last, want_last, 1e-11, "zero-order hold unrolled sum: last_state")


def pin_initial_state_free_decay(o):
    """u = 0 leaves only the start state: h_t,n = exp(A_n S_t) h0_n with S_t the running
    sum of Delta = softplus(delta + bias), so y_t = sum_n C_t,n exp(A_n S_t) h0_n."""
    rng = np.random.default_rng(35)
    batch, dim, N, L = 2, 3, 4, 30
    A = -rng.uniform(0.2, 2.0, (dim, N))
    h0 = rng.standard_normal((batch, dim, N))
    delta = rng.standard_normal((batch, dim, L))
    bias = rng.uniform(-1.0, 0.0, dim)
    C = rng.standard_normal((batch, N, L))
    B = rng.standard_normal((batch, N, L))
    D = rng.standard_normal(dim)
    u = np.zeros((batch, dim, L))
    S = np.cumsum(np.logaddexp(0.0, delta + bias[None, :, None]), axis=-1)   # (b, d, L)
    h = np.exp(A[None, :, :, None] * S[:, :, None, :]) * h0[..., None]        # (b, d, N, L)
    want = np.einsum("bdnt,bnt->bdt", h, C)
    for zoh in (False, True):
        out, last = o.selective_scan(u, delta, A, B, C, D=D, delta_bias=bias, softplus=True,
                                     zoh=zoh, initial_state=h0)
        _close(out, want, 1e-12, f"free decay from the start state (zoh={zoh}): out")
        _close(last, h[..., -1], 1e-12, f"free decay from the start state (zoh={zoh}): last")


def pin_initial_state_split(o):
    """A scan over L steps equals a scan over the first L1 steps followed by a scan over
    the rest that starts from the first part's last_state (both discretisations)."""
    p = _random_problem(36, seqlen=37)
    rng = np.random.default_rng(37)
    h0 = rng.standard_normal((2, 3, 4))
    z = rng.standard_normal(p["u"].shape)
    L1 = 15
    for zoh in (False, True):
        kw = dict(D=p["D"], delta_bias=p["delta_bias"], softplus=True, zoh=zoh)
        out, last = o.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], z=z,
                                     initial_state=h0, **kw)
        part = lambda a, sl: a[:, :, sl]
        o1, l1 = o.selective_scan(part(p["u"], slice(0, L1)), part(p["delta"], slice(0, L1)),
                                  p["A"], part(p["B"], slice(0, L1)), part(p["C"], slice(0, L1)),
                                  z=part(z, slice(0, L1)), initial_state=h0, **kw)
        o2, l2 = o.selective_scan(part(p["u"], slice(L1, None)), part(p["delta"], slice(L1, None)),
                                  p["A"], part(p["B"], slice(L1, None)),
                                  part(p["C"], slice(L1, None)), z=part(z, slice(L1, None)),
                                  initial_state=l1, **kw)
        _close(np.concatenate([o1, o2], axis=-1), out, 1e-13, f"split scan (zoh={zoh}): out")
        _close(l2, last, 1e-13, f"split scan (zoh={zoh}): last_state")


def pin_update_zoh(o):
    """Update with the zero-order hold: the Theorem-1 gate for N=1, A=-1, B=C=1, and
    T updates from a start state reproduce the zero-order-hold scan from that state."""
    rng = np.random.default_rng(38)
    batch, dim = 2, 5
    state = rng.standard_normal((batch, dim, 1))
    x = rng.standard_normal((batch, dim))
    dt = rng.standard_normal((batch, dim))
    bias = rng.uniform(-1.0, 1.0, dim)
    g = 1.0 / (1.0 + np.exp(-(dt + bias[None, :])))
    new, out = o.selective_state_update(state, x, dt, -np.ones((dim, 1)), np.ones((batch, 1)),
                                        np.ones((batch, 1)), dt_bias=bias, dt_softplus=True,
                                        zoh=True)
    gate = (1.0 - g) * state[:, :, 0] + g * x
    _close(new[:, :, 0], gate, 1e-13, "update zero-order hold gate: state")
    _close(out, gate, 1e-13, "update zero-order hold gate: out")
    p = _decode_problem(39)
    h0 = rng.standard_normal((2, 3, 4))
    out_scan, last = o.selective_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], D=p["D"],
                                      z=p["z"], delta_bias=p["bias"], softplus=True, zoh=True,
                                      initial_state=h0)
    st = h0.copy()
    outs = np.zeros_like(p["x"])
    for t in range(p["x"].shape[2]):
        st, outs[:, :, t] = o.selective_state_update(
            st, p["x"][:, :, t], p["dt"][:, :, t], p["A"], p["B"][:, :, t], p["C"][:, :, t],
            D=p["D"], z=p["z"][:, :, t], dt_bias=p["bias"], dt_softplus=True, zoh=True)
    _close(outs, out_scan, 1e-13, "zero-order-hold updates = scan: out")
    _close(st, last, 1e-13, "zero-order-hold updates = scan: state")


# ------------------------------------------------------------ short causal convolution
# "Mamba 与状态空间模型", 固定大小的状态: each channel keeps a short convolution
# over its 4 most recent inputs.  Conv state = the W most recent inputs, oldest first.

def _silu(v):
    return v / (1.0 + np.exp(-v))


def pin_conv_one_hot_is_a_delay(o):
    """A one-hot weight at tap k delays the input by W-1-k steps (zero before t = 0,
    the initial conv state when one is given)."""
    rng = np.random.default_rng(41)
    for W in (2, 3, 4):
        x = rng.standard_normal((2, 3, 11))
        init = rng.standard_normal((2, 3, W))
        for k in range(W):
            w = np.zeros((3, W))
            w[:, k] = 1.0
            lag = W - 1 - k
            out, _ = o.causal_conv1d(x, w, silu=False)
            want = np.concatenate([np.zeros((2, 3, lag)), x[:, :, :x.shape[2] - lag]], axis=2)
            _close(out, want, 0.0, f"conv delay W={W} k={k}")
            out, _ = o.causal_conv1d(x, w, initial_conv_state=init, silu=False)
            want = np.concatenate([init[:, :, W - lag:], x[:, :, :x.shape[2] - lag]], axis=2)
            _close(out, want, 0.0, f"conv delay from state W={W} k={k}")


def pin_conv_is_a_library_correlation(o):
    """out = silu(bias + correlate(state[1:] ++ x, w, 'valid')) per channel (numpy's
    correlation), and the final state is the last W inputs of state ++ x."""
    rng = np.random.default_rng(42)
    batch, dim, L, W = 2, 5, 23, 4
    x = rng.standard_normal((batch, dim, L))
    w = rng.standard_normal((dim, W))
    bias = rng.standard_normal(dim)
    init = rng.standard_normal((batch, dim, W))
    out, final = o.causal_conv1d(x, w, bias=bias, initial_conv_state=init, silu=True)
    want = np.zeros_like(x)
    want_final = np.zeros((batch, dim, W))
    for b in range(batch):
        for d in range(dim):
            xx = np.concatenate([init[b, d, 1:], x[b, d]])
            want[b, d] = _silu(np.correlate(xx, w[d], mode="valid") + bias[d])
            want_final[b, d] = np.concatenate([init[b, d], x[b, d]])[-W:]
    _close(out, want, 1e-13, "conv = library correlation")
    _close(final, want_final, 0.0, "conv final state")
    short, final_short = o.causal_conv1d(x[:, :, :2], w, initial_conv_state=init, silu=False)
    _close(final_short, np.concatenate([init, x[:, :, :2]], axis=2)[:, :, -W:], 0.0,
           "conv final state, L < W")


def pin_conv_silu_closed_values(o):
    """Identity tap, no bias: out = silu(x) at silu(0) = 0, silu(+-ln 3) = 3/4 ln 3,
    -1/4 ln 3, silu(40) = 40."""
    ln3 = math.log(3.0)
    x = np.array([0.0, ln3, -ln3, 40.0]).reshape(1, 1, 4)
    out, _ = o.causal_conv1d(x, np.array([[0.0, 0.0, 0.0, 1.0]]), silu=True)
    _close(out.reshape(-1), np.array([0.0, 0.75 * ln3, -0.25 * ln3, 40.0]), 1e-15,
           "conv silu closed values")


def pin_conv_updates_equal_prefill(o):
    """T single-token updates from a conv state reproduce the prefill convolution over
    the same T tokens from that state, outputs and final state; a prefill split in two
    equals the whole."""
    rng = np.random.default_rng(43)
    batch, dim, T, W = 3, 4, 9, 4
    x = rng.standard_normal((batch, dim, T))
    w = rng.standard_normal((dim, W))
    bias = rng.standard_normal(dim)
    init = rng.standard_normal((batch, dim, W))
    out, final = o.causal_conv1d(x, w, bias=bias, initial_conv_state=init, silu=True)
    st = init.copy()
    outs = np.zeros_like(x)
    for t in range(T):
        st, outs[:, :, t] = o.causal_conv1d_update(st, x[:, :, t], w, bias=bias, silu=True)
    _close(outs, out, 1e-14, "conv updates = prefill: out")
    _close(st, final, 0.0, "conv updates = prefill: state")
    o1, f1 = o.causal_conv1d(x[:, :, :4], w, bias=bias, initial_conv_state=init, silu=True)
    o2, f2 = o.causal_conv1d(x[:, :, 4:], w, bias=bias, initial_conv_state=f1, silu=True)
    _close(np.concatenate([o1, o2], axis=2), out, 1e-14, "conv split prefill: out")
    _close(f2, final, 0.0, "conv split prefill: state")


# ------------------------------------------------------------ backward pass
# "Mamba 与状态空间模型", 在芯片上扫过去: training back-propagates through the
# scan (recomputing the states).  The gradients are pinned to central finite
# differences of the forward oracle, which its own pins fix.

def _bwd_problem(seed, gated=True):
    rng = np.random.default_rng(seed)
    batch, dim, N, L = 2, 3, 3, 10
    p = dict(
        u=rng.standard_normal((batch, dim, L)),
        delta=rng.standard_normal((batch, dim, L)) * 0.7,
        A=-rng.uniform(0.3, 1.5, (dim, N)),
        B=rng.standard_normal((batch, N, L)) * 0.5,
        C=rng.standard_normal((batch, N, L)) * 0.5,
    )
    if gated:
        p.update(D=rng.standard_normal(dim), z=rng.standard_normal((batch, dim, L)),
                 delta_bias=rng.uniform(-0.5, 0.5, dim),
                 initial_state=rng.standard_normal((batch, dim, N)))
    dout = rng.standard_normal((batch, dim, L))
    dlast = rng.standard_normal((batch, dim, N)) if gated else None
    return p, dout, dlast


def _fd_check(o, p, dout, dlast, softplus, what, zoh=False):
    def loss(q):
        out, last = o.selective_scan(q["u"], q["delta"], q["A"], q["B"], q["C"], D=q.get("D"),
                                     z=q.get("z"), delta_bias=q.get("delta_bias"),
                                     softplus=softplus, initial_state=q.get("initial_state"),
                                     zoh=zoh)
        val = float(np.sum(dout * out))
        if dlast is not None:
            val += float(np.sum(dlast * last))
        return val

    g = o.selective_scan_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], dout, D=p.get("D"),
                             z=p.get("z"), delta_bias=p.get("delta_bias"), softplus=softplus,
                             initial_state=p.get("initial_state"), dlast_state=dlast, zoh=zoh)
    names = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
             "z": "dz", "delta_bias": "ddelta_bias", "initial_state": "dinitial_state"}
    for key, gname in names.items():
        if key not in p:
            assert gname not in g
            continue
        want = np.zeros_like(p[key])
        for idx in np.ndindex(p[key].shape):
            x0 = p[key][idx]
            eps = 1e-6 * max(1.0, abs(x0))
            q = {k: v.copy() for k, v in p.items()}
            q[key][idx] = x0 + eps
            lp = loss(q)
            q[key][idx] = x0 - eps
            lm = loss(q)
            want[idx] = (lp - lm) / (2 * eps)
        _close(g[gname], want, 2e-6, f"{what}: {gname} vs finite differences")


def pin_bwd_finite_differences_gated(o):
    """Every gradient (u, delta, A, B, C, D, z, bias, start state) with the gate,
    softplus, a start state and a last-state term, against central differences."""
    p, dout, dlast = _bwd_problem(51, gated=True)
    _fd_check(o, p, dout, dlast, True, "gated backward")


def pin_bwd_finite_differences_plain(o):
    """The same without gate, D, bias, start state or last-state term, softplus off."""
    p, dout, dlast = _bwd_problem(52, gated=False)
    _fd_check(o, p, dout, dlast, False, "plain backward")


def pin_bwd_zoh_finite_differences(o):
    """Zero-order-hold input term ("超越注意力：探索Mamba与状态空间模型", section
    状态空间模型基础: Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B): every gradient,
    gated, softplus on, with a start state and a last-state term, against central
    differences of the zero-order-hold forward.  One entry of A is set to 0
    (the gain's limit Delta) and one to -5e-4 (the series branch of dg/dA)."""
    p, dout, dlast = _bwd_problem(53, gated=True)
    p["A"][0, 0] = 0.0
    p["A"][1, 1] = -5e-4
    _fd_check(o, p, dout, dlast, True, "zero-order-hold backward", zoh=True)


def pin_bwd_zoh_plain_finite_differences(o):
    """The zero-order-hold backward without gate, D, bias, start state or
    last-state term, softplus off (Delta may then be negative)."""
    p, dout, dlast = _bwd_problem(54, gated=False)
    _fd_check(o, p, dout, dlast, False, "plain zero-order-hold backward", zoh=True)


# --- Mamba-2 layer (scalar A per head) ------------------------------------------------------
# "Mamba 与状态空间模型", section "Mamba-2：两种算法": with A a scalar times the identity,
# the layer is one lower-triangular matrix: entry (i, j) is C at step i dotted with B at
# step j, times all the decay between the two steps.  The pins below build that matrix
# (and the chunked / tied-diagonal readings of it) without stepping the recurrence.


def _ssd_problem(seed, batch=2, seqlen=23, nheads=4, headdim=3, ngroups=2, dstate=5,
                 with_state=True):
    rng = np.random.default_rng(seed)
    return dict(
        x=rng.standard_normal((batch, seqlen, nheads, headdim)),
        dt=rng.standard_normal((batch, seqlen, nheads)) * 0.5,
        A=-rng.uniform(0.3, 2.0, nheads),
        B=rng.standard_normal((batch, seqlen, ngroups, dstate)),
        C=rng.standard_normal((batch, seqlen, ngroups, dstate)),
        D=rng.standard_normal(nheads),
        z=rng.standard_normal((batch, seqlen, nheads, headdim)),
        dt_bias=rng.uniform(-1.0, 0.5, nheads),
        initial_state=(rng.standard_normal((batch, nheads, headdim, dstate))
                       if with_state else None),
    )


def _softplus(v):
    return np.log1p(np.exp(v))


def pin_ssd_lower_triangular_matrix(o):
    """out = (M x + start-state term + D x) * silu(z), M_ij = C_i.B_j exp(sum_{j<r<=i} Delta_r A) Delta_j."""
    p = _ssd_problem(41)
    out, final = o.ssd_scan(**p)
    batch, L, H, P = p["x"].shape
    G, N = p["B"].shape[2], p["B"].shape[3]
    delta = _softplus(p["dt"] + p["dt_bias"])             # (batch, L, H)
    for b in range(batch):
        for h in range(H):
            g = h // (H // G)
            a = delta[b, :, h] * p["A"][h]                    # log-decay of each step
            Bm, Cm = p["B"][b, :, g, :], p["C"][b, :, g, :]   # (L, N)
            M = np.zeros((L, L))
            for i in range(L):
                for j in range(i + 1):
                    M[i, j] = Cm[i] @ Bm[j] * math.exp(a[j + 1:i + 1].sum()) * delta[b, j, h]
            S0 = p["initial_state"][b, h]                     # (P, N)
            carry = np.array([math.exp(a[:i + 1].sum()) for i in range(L)])
            xs = p["x"][b, :, h, :]                           # (L, P)
            y = M @ xs + carry[:, None] * (Cm @ S0.T) + p["D"][h] * xs
            y = y * _silu(p["z"][b, :, h, :])
            _close(out[b, :, h, :], y, 1e-12, "SSD output vs the lower-triangular matrix")
            w = np.array([math.exp(a[j + 1:].sum()) * delta[b, j, h] for j in range(L)])
            S = math.exp(a.sum()) * S0 + (w[:, None] * xs).T @ Bm
            _close(final[b, h], S, 1e-12, "SSD final state vs the sum over steps")


def pin_ssd_is_tied_diagonal_scan(o):
    """One group: every (head, p) channel is a diagonal scan whose A row is A_h repeated."""
    p = _ssd_problem(42, ngroups=1, with_state=True)
    out, final = o.ssd_scan(**p)
    batch, L, H, P = p["x"].shape
    N = p["B"].shape[3]
    u = p["x"].transpose(0, 2, 3, 1).reshape(batch, H * P, L)
    z = p["z"].transpose(0, 2, 3, 1).reshape(batch, H * P, L)
    delta = np.repeat(p["dt"].transpose(0, 2, 1), P, axis=1)   # (batch, H*P, L)
    A = np.repeat(p["A"], P)[:, None] * np.ones((1, N))
    Bs = p["B"][:, :, 0, :].transpose(0, 2, 1)                # (batch, N, L)
    Cs = p["C"][:, :, 0, :].transpose(0, 2, 1)
    h0 = p["initial_state"].reshape(batch, H * P, N)
    ref_out, ref_last = o.selective_scan(u, delta, A, Bs, Cs, D=np.repeat(p["D"], P), z=z,
                                         delta_bias=np.repeat(p["dt_bias"], P),
                                         initial_state=h0)
    _close(out.transpose(0, 2, 3, 1).reshape(batch, H * P, L), ref_out, 1e-12,
           "SSD output vs the diagonal scan")
    _close(final.reshape(batch, H * P, N), ref_last, 1e-12, "SSD final state vs the diagonal scan")


def pin_ssd_split_equals_whole(o):
    """Scanning [0, k) then [k, L) from the first part's final state equals one scan."""
    p = _ssd_problem(43)
    out, final = o.ssd_scan(**p)
    k = 9
    first = {n: (v[:, :k] if n in ("x", "dt", "B", "C", "z") else v) for n, v in p.items()}
    second = {n: (v[:, k:] if n in ("x", "dt", "B", "C", "z") else v) for n, v in p.items()}
    out1, mid = o.ssd_scan(**first)
    second["initial_state"] = mid
    out2, final2 = o.ssd_scan(**second)
    _close(np.concatenate([out1, out2], axis=1), out, 1e-12, "SSD split output")
    _close(final2, final, 1e-12, "SSD split final state")


def pin_ssd_zero_A_is_cumulative_sum(o):
    """A = 0, softplus off, no gate, no D: S_t = S0 + sum_{j<=t} dt_j x_j B_j^T and y_t = S_t C_t."""
    p = _ssd_problem(44)
    p.update(A=np.zeros_like(p["A"]), dt=np.abs(p["dt"]), D=None, z=None, dt_bias=None)
    out, final = o.ssd_scan(**p, dt_softplus=False)
    batch, L, H, P = p["x"].shape
    G = p["B"].shape[2]
    for b in range(batch):
        for h in range(H):
            g = h // (H // G)
            terms = p["dt"][b, :, h, None, None] * np.einsum(
                "tp,tn->tpn", p["x"][b, :, h, :], p["B"][b, :, g, :])
            S = p["initial_state"][b, h][None] + np.cumsum(terms, axis=0)   # (L, P, N)
            y = np.einsum("tpn,tn->tp", S, p["C"][b, :, g, :])
            _close(out[b, :, h, :], y, 1e-12, "SSD with A = 0 vs the cumulative sum")
            _close(final[b, h], S[-1], 1e-12, "SSD with A = 0, final state")


PINS = {
    "unrolled_sum": pin_unrolled_sum,
    "gate_closed_values": pin_gate_closed_values,
    "lti_convolution": pin_lti_convolution,
    "gated_rnn_theorem1": pin_gated_rnn_theorem1,
    "small_delta_holds": pin_small_delta_holds,
    "large_delta_resets": pin_large_delta_resets,
    "zero_A_cumulative_sum": pin_zero_A_cumulative_sum,
    "softplus_closed_values": pin_softplus_closed_values,
    "linearity_and_causality": pin_linearity_and_causality,
    "update_steps_equal_scan": pin_update_steps_equal_scan,
    "update_continues_scan": pin_update_continues_scan,
    "update_limits": pin_update_limits,
    "zoh_gated_rnn_exact": pin_zoh_gated_rnn_exact,
    "zoh_fixed_point": pin_zoh_fixed_point,
    "zoh_zero_A_is_cumulative_sum": pin_zoh_zero_A_is_cumulative_sum,
    "zoh_unrolled_sum": pin_zoh_unrolled_sum,
    "initial_state_free_decay": pin_initial_state_free_decay,
    "initial_state_split": pin_initial_state_split,
    "update_zoh": pin_update_zoh,
    "conv_one_hot_is_a_delay": pin_conv_one_hot_is_a_delay,
    "conv_is_a_library_correlation": pin_conv_is_a_library_correlation,
    "conv_silu_closed_values": pin_conv_silu_closed_values,
    "conv_updates_equal_prefill": pin_conv_updates_equal_prefill,
    "bwd_finite_differences_gated": pin_bwd_finite_differences_gated,
    "bwd_finite_differences_plain": pin_bwd_finite_differences_plain,
    "bwd_zoh_finite_differences": pin_bwd_zoh_finite_differences,
    "bwd_zoh_plain_finite_differences": pin_bwd_zoh_plain_finite_differences,
    "ssd_lower_triangular_matrix": pin_ssd_lower_triangular_matrix,
    "ssd_is_tied_diagonal_scan": pin_ssd_is_tied_diagonal_scan,
    "ssd_split_equals_whole": pin_ssd_split_equals_whole,
    "ssd_zero_A_is_cumulative_sum": pin_ssd_zero_A_is_cumulative_sum,
}
