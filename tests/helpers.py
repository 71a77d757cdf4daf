"""Tolerances of the GPU-vs-oracle comparisons.

* logZ: relative 1e-5 with an absolute floor at the log path count,
  |d| <= 1e-5 * max(|logZ_ref|, (L + D(n-1)) ln 2)  (logZ passes near 0 at
  moderate T, where a pure relative bound is meaningless);
* soft codeword: |d| <= 1e-5 * max|c|;
* gradients: max|d| <= 1e-4 * max|g_ref| per tensor (relative 1e-4 read as a
  max-norm bound);
* Viterbi states and costs: bit-exact.
"""
import math

import numpy as np


def logZ_tol(ref, L, D, n):
    floor = (L + D * (n - 1)) * math.log(2.0)
    return 1e-5 * np.maximum(np.abs(np.asarray(ref, np.float64)), floor)


def assert_logZ(gpu, ref, L, D, n):
    gpu = np.asarray(gpu, np.float64); ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref)
    tol = logZ_tol(ref, L, D, n)
    bad = err > tol
    assert not bad.any(), f"logZ: {bad.sum()} violations, worst err {err.max():.3e} (tol {tol.min():.3e})"


def assert_soft(gpu, ref, c):
    gpu = np.asarray(gpu, np.float64); ref = np.asarray(ref, np.float64)
    tol = 1e-5 * float(np.abs(np.asarray(c, np.float64)).max())
    err = np.abs(gpu - ref).max()
    assert err <= tol, f"soft codeword: max err {err:.3e} > tol {tol:.3e}"


def assert_grad(gpu, ref, name="grad"):
    gpu = np.asarray(gpu, np.float64); ref = np.asarray(ref, np.float64)
    scale = float(np.abs(ref).max())
    err = float(np.abs(gpu - ref).max())
    assert err <= 1e-4 * scale, f"{name}: max err {err:.3e} > 1e-4 * {scale:.3e}"


def unique_argmax_mask(top2, margin=1e-4):
    """Steps whose oracle posterior argmax is unique by a margin."""
    return (top2[..., 0] - top2[..., 1]) > margin
