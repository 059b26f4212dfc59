"""Shared helpers for the GPU parity tests (error metrics and the stated tolerance)."""
import numpy as np

# Tolerance of the method's target: bf16 inputs, fp32 accumulation, bf16 output, compared with
# the fp64 oracle element by element.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU output"
    d = np.abs(got - ref)
    return float(d.max()), float(d.mean())


def assert_close(got, ref, what=""):
    mx, mn = errors(got, ref)
    assert mx <= MAX_ABS and mn <= MEAN_ABS, f"{what}: max|err| {mx:.3e} mean|err| {mn:.3e}"
    return mx, mn
