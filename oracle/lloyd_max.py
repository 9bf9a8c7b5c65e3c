"""16-level Lloyd-Max codebook for N(0, 1) -- oracle (test infrastructure).

What the pages fix:
- OrbitQuant PR #25, "Default changes": activations below 8 bits use Lloyd-Max codes; the
  codebook solver moved from an iteration (v2) to Newton (v3).
- CentriQ §2 (related work on OrbitQuant): the codebook is derived from the post-rotation
  marginal. After per-token normalisation that marginal is modelled as N(0, 1), the d -> inf
  limit of the finite-width marginal.

This oracle runs the classical Lloyd (1957/1982) / Max (1960) fixed-point iteration, which is
the definition of a Lloyd-Max quantizer: thresholds at the midpoints of adjacent centroids,
centroids at the conditional means of their cells,
    tau_k = (c_k + c_{k+1}) / 2,
    c_k   = (phi(tau_{k-1}) - phi(tau_k)) / (Phi(tau_k) - Phi(tau_{k-1})),
with tau_{-1} = -inf and tau_{L-1} = +inf. The library solves the same conditions with
Newton's method; the two are independent.

Parity: pinned (tests/test_oracle_lloyd_max.py): both optimality conditions, symmetry, the
mean-squared error Max (1960) tabulates for 16 levels, and agreement with a direct numerical
minimisation of the distortion by scipy.optimize.
"""
from __future__ import annotations

import numpy as np
from scipy.special import ndtr

_INV_SQRT_2PI = 1.0 / np.sqrt(2.0 * np.pi)


def _phi(x: np.ndarray) -> np.ndarray:
    out = np.zeros_like(x)
    fin = np.isfinite(x)
    out[fin] = np.exp(-0.5 * x[fin] ** 2) * _INV_SQRT_2PI
    return out


def _cell_prob(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Phi(b) - Phi(a), evaluated on the side of zero that keeps precision."""
    left = ndtr(b) - ndtr(a)
    right = ndtr(-a) - ndtr(-b)
    return np.where(a >= 0.0, right, left)


def lloyd_max_gaussian(levels: int = 16, tol: float = 1e-15, max_iter: int = 200000):
    """Return (centroids[levels], thresholds[levels-1]) of the N(0,1) Lloyd-Max quantizer."""
    c = np.linspace(-2.5, 2.5, levels)
    for _ in range(max_iter):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate(([-np.inf], t, [np.inf]))
        p = _cell_prob(edges[:-1], edges[1:])
        c_new = (_phi(edges[:-1]) - _phi(edges[1:])) / p
        if np.max(np.abs(c_new - c)) < tol:
            c = c_new
            break
        c = c_new
    t = 0.5 * (c[:-1] + c[1:])
    return c, t


def lloyd_max_mse(centroids: np.ndarray, thresholds: np.ndarray) -> float:
    """Distortion E[(X - Q(X))^2] for X ~ N(0, 1), by the cell-wise closed form.

    For a cell [a, b] with reconstruction c:  int (x - c)^2 phi = (Phi(b) - Phi(a)) (1 + c^2)
    + a phi(a) - b phi(b) - 2 c (phi(a) - phi(b)), with x phi(x) -> 0 at +-inf.
    """
    edges = np.concatenate(([-np.inf], thresholds, [np.inf]))
    a, b = edges[:-1], edges[1:]
    p = _cell_prob(a, b)
    pa, pb = _phi(a), _phi(b)
    with np.errstate(invalid="ignore"):
        apa = np.where(np.isfinite(a), a * pa, 0.0)
        bpb = np.where(np.isfinite(b), b * pb, 0.0)
    second = p + apa - bpb                   # int x^2 phi over the cell
    first = pa - pb                          # int x phi over the cell
    return float(np.sum(second - 2.0 * centroids * first + centroids ** 2 * p))
