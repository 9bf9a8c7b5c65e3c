"""Asymmetric grouped INT4 weights -- oracle (test infrastructure).

What the pages fix (CentriQ: Calibration-Free Quantization of Diffusion Transformers via Exact
Mean Centering):
- §3, Eq. 2: weights are quantized to an asymmetric b-bit grid over groups of g consecutive
  input columns, W_g = sigma (Q_g - z), Q_g in {0, ..., 2^b - 1}, with a per-(row, group)
  scale sigma and shift z stored in 16 bits; round to nearest (RTN) sets both from the group
  minimum and maximum.
- §4.3: the groups are g = 64 consecutive columns of the rotated weight W_R = W Q^T; row i of
  group g reconstructs as s_i sigma_ig (Q_ig - z_ig) with a per-row scale s_i (1 under RTN).
- App. B.2: codes are stored as Q - 8 with zero point z' = z - 8, which leaves a correction
  C = sigma z' per row and group; with p_t,g the group sums of the activation codes the
  product is sum_g sigma_g (sum_{k in g} a_k (Q_k - 8) - z'_g p_t,g).
- App. B.3, Tab. 3: grid {0..15}, g = 64, scale and zero point in FP16 (PixArt-Sigma) or BF16.

Readings: sigma = max(max - min, eps) / (2^b - 1) and z = -min / sigma (HQQ-style min/max
initialisation with a real shift); with 16-bit storage sigma and z are rounded to fp16 (the
format of the tensor-core operand) and the codes are taken against the stored grid,
Q = clip(round(w / sigma16 + z16), 0, 2^b - 1), round half to even. Before rounding, sigma is
floored at 2^-14 (the smallest normal fp16, so that the stored grid never degenerates) and at
|min| / 2^15, so that the stored shift |z| = |min| / sigma16 stays below 2^15 (1 + 2^-11) and
is finite in fp16 even for a nearly constant group far from zero; the grid still covers
[min, max] because 15 sigma >= max - min. The activations that multiply these weights are the
INT4 absmax (or percentile) codes.

Parity: pinned (tests/test_oracle_weights_g64.py): the reconstruction error is at most
sigma / 2 everywhere, group minima and maxima reconstruct exactly (exact storage), the codes
equal a brute-force nearest point of the stored grid, and the zero-point correction of App. B.2
equals the dequantized product.
"""
from __future__ import annotations

import numpy as np

from .linear import epilogue, quantize_activations
from .quant import EPS
from .rpbh import rotate

GROUP = 64
SIGMA_MIN_F16 = 2.0 ** -14
SHIFT_MAX = 2.0 ** 15      # 16-bit storage: sigma >= |min| / SHIFT_MAX keeps z finite


def asym_group_quantize(w: np.ndarray, g: int = GROUP, bits: int = 4, store=None,
                        eps: float = EPS):
    """Per (row, group of g columns): (codes Q int64 [N, d] in 0..2^b-1, sigma [N, d/g],
    z [N, d/g]) with W_hat = sigma (Q - z). ``store=np.float16`` rounds sigma (floored at
    2^-14) and z to fp16 first and codes against the stored grid; None keeps them exact."""
    w = np.asarray(w, dtype=np.float64)
    n, d = w.shape
    if d % g:
        raise ValueError("d must be a multiple of the group size")
    top = 2 ** bits - 1
    wg = w.reshape(n, d // g, g)
    lo, hi = wg.min(axis=2), wg.max(axis=2)
    sigma = np.maximum(hi - lo, eps) / top
    if store is not None:
        sigma = np.maximum(np.maximum(sigma, SIGMA_MIN_F16), np.abs(lo) / SHIFT_MAX)
        sigma = sigma.astype(store).astype(np.float64)
    z = -lo / sigma
    if store is not None:
        z = z.astype(store).astype(np.float64)
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


def prepare_weights_g64(w: np.ndarray, plan, h: int):
    """W_R = W Q^T (rows rotated, no centering), asymmetric INT4 groups of 64 with fp16 sigma
    and z, and w_1 = W 1. Returns (Q int64 [N, d], sigma [N, d/64], z [N, d/64], w_1 [N])."""
    w = np.asarray(w, dtype=np.float64)
    q, sigma, z = asym_group_quantize(rotate(w, plan, h), store=np.float16)
    return q, sigma, z, w.sum(axis=1)


def linear_forward_g64(x, w, plan, h, act, center_tokens, bias=None):
    """The layer with INT4 absmax (or percentile) activations against asymmetric g = 64
    weights, in float64: y = alpha_t sum_k a_k W_hat[o, k] + mean_t w_1[o] + b[o] (s_i = 1).
    Returns (y, activation dict, (Q, sigma, z, w_1))."""
    qa = quantize_activations(x, plan, h, act, center_tokens)
    q, sigma, z, w1 = prepare_weights_g64(w, plan, h)
    acc = np.asarray(qa["codes"], np.float64) @ dequantize(q, sigma, z).T
    y = epilogue(acc, qa["scale"], np.ones(q.shape[0]), qa["mean"] if center_tokens else None,
                 w1 if center_tokens else None, bias)
    return y, qa, (q, sigma, z, w1)
