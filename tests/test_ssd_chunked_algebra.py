"""The chunked algebra of the Mamba-2 layer kernel, checked on the CPU in float64.

The tensor-core kernel does not step the recurrence: per chunk of Q tokens it
forms the running log2-decay c, the matrices G = C B^T and
Gm_ij = G_ij 2^(c_i - c_j) Delta_j (j <= i) plus D_h on the diagonal, the
entering state's read-out 2^(c_i) C H^T, the weighted input
Xw_j = 2^(c_Q - c_j) Delta_j x_j and the new state 2^(c_Q) H + (B^T Xw)^T.
This test writes those steps out in numpy without any rounding and requires
them to reproduce the float64 oracle's recurrence to 1e-12 for several chunk
lengths, groups, a start state and a ragged last chunk ("Mamba 与状态空间模型",
section "Mamba-2：两种算法": matrix products inside a chunk, only the state
passed between chunks)."""
import numpy as np
import pytest

from oracle import oracle


def _problem(seed, batch=2, L=45, H=4, P=3, G=2, N=5):
    rng = np.random.default_rng(seed)
    return dict(
        x=rng.standard_normal((batch, L, H, P)),
        dt=rng.standard_normal((batch, L, H)) * 0.5,
        A=-rng.uniform(0.3, 2.0, H),
        B=rng.standard_normal((batch, L, G, N)),
        C=rng.standard_normal((batch, L, G, N)),
        D=rng.standard_normal(H),
        z=rng.standard_normal((batch, L, H, P)),
        dt_bias=rng.uniform(-1.0, 0.5, H),
        initial_state=rng.standard_normal((batch, H, P, N)),
    )


def _chunked(p, Q):
    x, dt, A, B, C, D, z = (p[k] for k in ("x", "dt", "A", "B", "C", "D", "z"))
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    delta = np.log1p(np.exp(dt + p["dt_bias"]))
    out = np.zeros_like(x)
    final = np.zeros((batch, H, P, N))
    for b in range(batch):
        for h in range(H):
            g = h // (H // G)
            S = p["initial_state"][b, h].copy()                     # (P, N)
            for l0 in range(0, L, Q):
                sl = slice(l0, min(L, l0 + Q))
                Cc, Bc, Xc, dl = C[b, sl, g], B[b, sl, g], x[b, sl, h], delta[b, sl, h]
                c = np.cumsum(dl * A[h]) / np.log(2.0)              # log2-decay
                G_ = Cc @ Bc.T
                Gm = np.tril(G_ * np.exp2(c[:, None] - c[None, :]) * dl[None, :])
                Gm += D[h] * np.eye(len(dl))
                y = Gm @ Xc + np.exp2(c)[:, None] * (Cc @ S.T)
                out[b, sl, h] = y * z[b, sl, h] / (1.0 + np.exp(-z[b, sl, h]))
                Xw = (np.exp2(c[-1] - c) * dl)[:, None] * Xc
                S = np.exp2(c[-1]) * S + (Bc.T @ Xw).T
            final[b, h] = S
    return out, final


@pytest.mark.parametrize("Q", [1, 4, 7, 16, 128])
def test_chunked_steps_equal_the_recurrence(Q):
    p = _problem(7)
    ref = oracle.default()
    o_out, o_final = ref.ssd_scan(**p)
    out, final = _chunked(p, Q)
    scale_o = np.max(np.abs(o_out))
    scale_f = np.max(np.abs(o_final))
    assert np.max(np.abs(out - o_out)) <= 1e-12 * scale_o
    assert np.max(np.abs(final - o_final)) <= 1e-12 * scale_f
