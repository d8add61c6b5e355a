"""Gaussian Lloyd-Max quantizer levels.

"E22L" "Result" (last paragraphs) names the value grid to test next after the ggml signed
2-bit grid: a symmetric grid, or Lloyd-Max levels for a Gaussian applied after rotation.  The pages give
no table.  This builds the levels from their definition (the MSE-optimal fixed-rate quantizer
of a density; S. P. Lloyd, "Least squares quantization in PCM", and J. Max, "Quantizing for
minimum distortion", 1960): at the optimum every threshold is the midpoint of its two
neighbouring levels, and every level is the centroid of its cell.  For the standard normal
density phi with distribution Phi the centroid of (a, b] is (phi(a) - phi(b)) / (Phi(b) - Phi(a)).
Starting from evenly spaced levels, the two conditions are applied in turn (Lloyd's iteration)
until the levels stop moving, in fp64.

Reading taken here (as for NF4): the levels are stored at fp16 precision, so a level times an
fp16 scale is exact in fp32 and the decision thresholds (midpoints times the scale) are exact.
The group scale is the group's root-mean-square value (the standard deviation of the zero-mean
Gaussian the levels assume).
"""
from __future__ import annotations

import math

import numpy as np


def _phi(x: np.ndarray) -> np.ndarray:
    return np.where(np.isinf(x), 0.0, np.exp(-0.5 * np.where(np.isinf(x), 0.0, x) ** 2) / math.sqrt(2 * math.pi))


def _Phi(x: np.ndarray) -> np.ndarray:
    return np.array([0.5 * math.erfc(-v / math.sqrt(2.0)) for v in x])


def centroids(thresholds: np.ndarray) -> np.ndarray:
    """E[X | t_(k-1) < X <= t_k] of the standard normal for the cells the thresholds bound."""
    lo = np.concatenate([[-np.inf], thresholds])
    hi = np.concatenate([thresholds, [np.inf]])
    return (_phi(lo) - _phi(hi)) / (_Phi(hi) - _Phi(lo))


def lloyd_max_levels_f64(bits: int, tol: float = 1e-12, max_iter: int = 200000) -> np.ndarray:
    n = 2 ** bits
    lv = np.linspace(-2.0, 2.0, n)
    for _ in range(max_iter):
        new = centroids((lv[:-1] + lv[1:]) / 2.0)
        if np.abs(new - lv).max() < tol:
            return new
        lv = new
    raise RuntimeError("Lloyd iteration did not settle")


_CACHE: dict = {}


def lloyd_max_levels(bits: int) -> np.ndarray:
    """The 2^bits sorted levels (units of the standard deviation) as fp16 values in fp64."""
    if bits not in _CACHE:
        _CACHE[bits] = lloyd_max_levels_f64(bits).astype(np.float16).astype(np.float64)
    return _CACHE[bits]
