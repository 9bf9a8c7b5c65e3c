"""Asymmetric grouped INT4 weights -- oracle (test infrastructure).

What the pages fix (CentriQ: Calibration-Free Quantization of Diffusion Transformers via Exact
Mean Centering):
- §3, Eq. 2: weights are quantized to an asymmetric b-bit grid over groups of g consecutive
  input columns, W_g = sigma (Q_g - z), Q_g in {0, ..., 2^b - 1}, with a per-(row, group)
  scale sigma and shift z.
- §4.3: the groups are g = 64 consecutive columns of the rotated weight W_R = W Q^T; round to
  nearest (RTN) sets the scale and the shift from the group minimum and maximum.
- App. B.2: codes are stored as Q - 8 with zero point z' = z - 8, which leaves a correction
  C = sigma z' per row and group; with p_t,g the group sums of the activation codes the
  product is sum_g sigma_g (sum_{k in g} a_k (Q_k - 8) - z'_g p_t,g).

Readings: sigma = max(max - min, eps) / (2^b - 1) and z = -min / sigma (a real shift, so that
the group minimum and maximum reconstruct exactly); Q = clip(round(w / sigma + z), 0, 2^b - 1)
with round half to even; the activations multiplying these weights are the A4 absmax codes.

Parity: pinned (tests/test_oracle_weights_g64.py): the reconstruction error is at most
sigma / 2 everywhere, group minima and maxima reconstruct exactly, the codes equal a brute-force
nearest grid point on small groups, and the zero-point correction of App. B.2 equals the
dequantized product.
"""
from __future__ import annotations

import numpy as np

from .quant import EPS

GROUP = 64


def asym_group_quantize(w: np.ndarray, g: int = GROUP, bits: int = 4, eps: float = EPS):
    """Per (row, group of g columns): (codes Q int64 [N, d] in 0..2^b-1, sigma [N, d/g],
    z [N, d/g]) with W_hat = sigma (Q - z)."""
    w = np.asarray(w, dtype=np.float64)
    n, d = w.shape
    if d % g:
        raise ValueError("d must be a multiple of the group size")
    top = 2 ** bits - 1
    wg = w.reshape(n, d // g, g)
    lo, hi = wg.min(axis=2), wg.max(axis=2)
    sigma = np.maximum(hi - lo, eps) / top
    z = -lo / sigma
    q = np.clip(np.rint(wg / sigma[..., None] + z[..., None]), 0, top).astype(np.int64)
    return q.reshape(n, d), sigma, z


def dequantize(q: np.ndarray, sigma: np.ndarray, z: np.ndarray, g: int = GROUP) -> np.ndarray:
    """W_hat = sigma (Q - z) per group (float64)."""
    n, d = q.shape
    qg = np.asarray(q, dtype=np.float64).reshape(n, d // g, g)
    return (sigma[..., None] * (qg - z[..., None])).reshape(n, d)


def corrected_product(a_codes: np.ndarray, q: np.ndarray, sigma: np.ndarray, z: np.ndarray,
                      g: int = GROUP) -> np.ndarray:
    """App. B.2: sum_g sigma_g (sum_{k in g} a_k (Q_k - 8) - z'_g p_g) with z' = z - 8 and
    p_g the group sums of the activation codes. [T, N] float64."""
    a = np.asarray(a_codes, dtype=np.float64)
    t, d = a.shape
    n = q.shape[0]
    ag = a.reshape(t, d // g, g)
    qs = (np.asarray(q, dtype=np.float64) - 8.0).reshape(n, d // g, g)
    main = np.einsum("tgk,ngk->tng", ag, qs)          # integer products per group
    p = ag.sum(axis=2)                                 # [T, G]
    corr = (z - 8.0)[None, :, :] * p[:, None, :]       # z'_g p_t,g
    return np.einsum("tng,ng->tn", main - corr, sigma)
