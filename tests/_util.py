"""Shared helpers for the test suite (comparison metrics and tolerances)."""

import numpy as np

# Decode-output tolerance: max|delta| <= 2e-2 * max|ref| and
# sum|delta| / sum|ref| <= 5e-3, for bf16 operands with fp32 accumulation.
TOL_MAX = 2e-2
TOL_MEAN = 5e-3


def parity_metrics(got, ref):
    """(max|got-ref| / max|ref|, sum|got-ref| / sum|ref|) over all elements."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in result"
    d = np.abs(got - ref)
    return float(d.max() / np.abs(ref).max()), float(d.sum() / np.abs(ref).sum())


def assert_parity(got, ref, what="", tol_max=TOL_MAX, tol_mean=TOL_MEAN):
    mx, mean = parity_metrics(got, ref)
    assert mx <= tol_max and mean <= tol_mean, (
        f"{what}: max|d|/max|ref| = {mx:.3e} (tol {tol_max}), "
        f"sum|d|/sum|ref| = {mean:.3e} (tol {tol_mean})")
    return mx, mean
