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

Per-width codebooks (OrbitQuant PR #25: "codebook v3" solves a table per width d; CentriQ
§2: the codebook is derived from the post-rotation marginal). Reading: after a rotation that
leaves the token's direction uniform on the sphere, one coordinate of the token normalised to
unit RMS is y = sqrt(d) u_1 with u uniform on S^(d-1), whose density is
    f_d(y) = c_d (1 - y^2 / d)^((d - 3) / 2)  on |y| < sqrt(d),
    c_d = Gamma(d / 2) / (sqrt(pi d) Gamma((d - 1) / 2)),
which tends to N(0, 1) as d grows. Its cell probabilities are regularized incomplete beta
functions (u_1^2 ~ Beta(1/2, (d - 1)/2)) and its first moment over a cell has the closed form
int_a^b y f_d(y) dy = m_d(a) - m_d(b), m_d(t) = c_d d / (d - 1) (1 - t^2 / d)^((d - 1) / 2).
The same Lloyd iteration runs on f_d.

Parity: pinned (tests/test_oracle_lloyd_max.py): both optimality conditions, symmetry, the
mean-squared error Max (1960) tabulates for 16 levels, and agreement with a direct numerical
minimisation of the distortion by scipy.optimize. Per-width tables: d = 3 gives the uniform
density, whose Lloyd-Max quantizer is the uniform one (closed form); the centroid and midpoint
conditions checked by adaptive quadrature of f_d itself; large d approaching the N(0, 1)
table; and the distortion against a Monte Carlo of random directions.
"""
from __future__ import annotations

import functools

import numpy as np
from scipy.special import betainc, gammaln, ndtr

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


def sphere_marginal(d: int):
    """(pdf, cdf, first-moment tail m) of y = sqrt(d) u_1, u uniform on S^(d-1)."""
    r = np.sqrt(float(d))
    log_c = gammaln(d / 2.0) - 0.5 * np.log(np.pi * d) - gammaln((d - 1) / 2.0)

    def pdf(y):
        y = np.asarray(y, dtype=np.float64)
        inside = np.abs(y) < r
        out = np.zeros_like(y)
        out[inside] = np.exp(log_c + 0.5 * (d - 3) * np.log1p(-y[inside] ** 2 / d))
        return out

    def cdf(y):
        y = np.clip(np.asarray(y, dtype=np.float64), -r, r)
        return 0.5 + 0.5 * np.sign(y) * betainc(0.5, 0.5 * (d - 1), np.minimum(y * y / d, 1.0))

    def m(y):
        y = np.clip(np.asarray(y, dtype=np.float64), -r, r)
        return np.exp(log_c) * d / (d - 1.0) * np.power(np.maximum(1.0 - y * y / d, 0.0),
                                                        0.5 * (d - 1))

    return pdf, cdf, m


def lloyd_max_sphere(d: int, levels: int = 16, tol: float = 1e-15, max_iter: int = 200000):
    """(centroids, thresholds) of the Lloyd-Max quantizer for the width-d marginal f_d."""
    if d < 3:
        raise ValueError("d >= 3")
    _, cdf, m = sphere_marginal(d)
    r = np.sqrt(float(d))
    c = np.linspace(-0.9, 0.9, levels) * min(2.5, 0.9 * r)
    for _ in range(max_iter):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate(([-r], t, [r]))
        p = cdf(edges[1:]) - cdf(edges[:-1])
        c_new = (m(edges[:-1]) - m(edges[1:])) / p
        if np.max(np.abs(c_new - c)) < tol:
            c = c_new
            break
        c = c_new
    return c, 0.5 * (c[:-1] + c[1:])


@functools.lru_cache(maxsize=None)
def lloyd_max_gaussian_8bit():
    """(centroids[256], thresholds[255]) of the 256-level N(0, 1) Lloyd-Max quantizer (the
    A8 Lloyd-Max codes of OrbitQuant PR #25's comparison). Lloyd's iteration converges slowly
    at 256 levels; it stops when no centroid moves by 1e-13."""
    c, t = lloyd_max_gaussian(levels=256, tol=1e-13, max_iter=2000000)
    c.setflags(write=False)
    t.setflags(write=False)
    return c, t

