"""Error metric and tolerances for comparing the CUDA path with the oracle.

err = max_i |got_i - want_i| / max(|want_i|, rms(want)).  The denominator is
the element's own magnitude, floored at the RMS of the reference so that
elements near zero (an output gated by silu(z) ~ 0) do not divide by ~0.

Tolerances: 1e-5 for fp32 inputs and outputs; 2e-2 for bf16 inputs/outputs
with the fp32 state (the bf16 rounding of the output alone is up to 2^-9).
"""
import numpy as np
import torch

FP32_TOL = 1e-5
BF16_TOL = 2e-2


def as_f64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def max_rel_err(got, want) -> float:
    """The error metric above; infinity when either side holds a non-finite
    value, so that a NaN can never pass a tolerance."""
    got, want = as_f64(got), as_f64(want)
    assert got.shape == want.shape, (got.shape, want.shape)
    if want.size == 0:
        return 0.0
    if not (np.all(np.isfinite(got)) and np.all(np.isfinite(want))):
        return float("inf")
    rms = float(np.sqrt(np.mean(want * want)))
    denom = np.maximum(np.abs(want), rms)
    denom = np.where(denom > 0, denom, 1.0)
    return float(np.max(np.abs(got - want) / denom))


def tol_for(dtype) -> float:
    return FP32_TOL if dtype == torch.float32 else BF16_TOL


# A second, componentwise bound for the Mamba-2 layer on the tensor cores: the
# same recurrence run on the absolute values of the inputs gives, per element,
# the sum of the magnitudes of every term that reaches it, and the error must
# stay below SCALED_TOL times that sum.  The kernel carries each operand it
# computes (the masked intra-chunk matrix, the state copy, the weighted input)
# as a bf16 hi/lo pair, good to about 2^-17, so the bf16 rounding of the output
# (2^-9 of |output|, which the sum bounds) is the only rounding at that level;
# SCALED_TOL = 2^-8 leaves a factor of two.  The layer's tests apply it beside
# the max_rel_err gate above (2e-2 for bf16 inputs with the fp32 state).
SCALED_TOL = 2.0 ** -8


def max_scaled_err(got, want, scale) -> float:
    """max_i |got_i - want_i| / scale_i (scale_i floored at 1e-30); infinity
    when either side holds a non-finite value."""
    got, want, scale = as_f64(got), as_f64(want), as_f64(scale)
    assert got.shape == want.shape == scale.shape, (got.shape, want.shape, scale.shape)
    if want.size == 0:
        return 0.0
    if not (np.all(np.isfinite(got)) and np.all(np.isfinite(want))):
        return float("inf")
    return float(np.max(np.abs(got - want) / np.maximum(scale, 1e-30)))
