"""Per-token centering and quantizers -- oracle (test infrastructure).

What the pages fix:
- CentriQ §3, Eq. 1: symmetric b-bit per-token quantizer,
  Q_a(x) = alpha * clip(round(x / alpha), -(2^(b-1) - 1), 2^(b-1) - 1), alpha = r / (2^(b-1) - 1),
  with range r = ||x||_inf (absmax). b = 8 gives the A8 grid {-127..127}; b = 4 gives
  {-7..7} (App. B.2: "quantizes to {-7,...,7}"); b = 2 gives the ternary A2 grid {-1, 0, 1},
  the activation grid of CentriQ's W4A2 configuration (App. B.3, Tab. 3: one grid formula for
  every b; App. C.1, Tab. 4: W4A2 on FLUX.1-schnell).
- OrbitQuant PR #25, "Default changes": absmax INT8 at A8, Lloyd-Max codes below.
- CentriQ §4.2 "Centering and exact re-injection": x_c = x - mean(x) * 1 over the n native
  channels, one scalar stored beside the per-token scale.
- FLUX.1-schnell-OrbitQuant-W4A4 model card, "Quantization": activation normalization
  epsilon 1e-10.
- CentriQ §4.2 "Scale and grid" and App. B.3 (Tab. 3): the percentile scale. The spread of the
  rotated token is sigma_hat = q_rho(|z|) / Phi^-1((1 + rho) / 2), the empirical rho-quantile
  of the magnitudes over the half-normal quantile, and alpha = gamma * sigma_hat / (2^(b-1) - 1)
  with rho = 0.9995 and gamma = 2.5591 (Tab. 3; §4.2 rounds it to 2.56), values beyond the
  range clipping to the end of the grid.

Readings where the pages are open:
- round() is round-half-to-even; the range is floored at eps: alpha = max(r, eps) / qmax.
- The Lloyd-Max scale is the token's RMS, sigma = max(sqrt(mean(z^2)), eps), which normalises
  the rotated token to the unit-variance marginal the N(0, 1) codebook is built for.
  The code of a value u = z / sigma is the number of thresholds strictly below u (nearest
  centroid; a tie at a threshold goes to the lower index).
- 4-bit codes are packed two per byte: element 2j in bits 0-3 of byte j, element 2j+1 in
  bits 4-7. Absmax codes are two's-complement nibbles; Lloyd-Max codes are indices 0..15.
- 2-bit codes (A2) are packed four per byte: element 4j + i in bits 2i, 2i + 1 of byte j, as
  two's-complement pairs (-1 is 0b11). The pages only simulate A2 (CentriQ §7: no fused
  kernel supports 2-bit activations yet), so they fix no storage; this is the plainest one.
- A2 takes the percentile range only: CentriQ's W4A2 results use its percentile scale
  (Tab. 3 gives the quantile and clip for all activation widths).
- The percentile scale's "empirical quantile" is the linear interpolation between order
  statistics at position rho (n - 1) (NumPy's and PyTorch's default); its range
  gamma * sigma_hat takes the same eps floor as the absmax range.

Parity: pinned (tests/test_oracle_quant.py): the largest coordinate maps to +-qmax, the
error bound |z - alpha q| <= alpha / 2, brute-force nearest grid point on small inputs,
nearest-centroid brute force for Lloyd-Max codes, offset invariance of centered codes
(CentriQ Eq. 6), pack/unpack round trips and hand-written byte examples (nibbles and 2-bit
pairs); the ternary grid (b = 2) against its closed form sign(z) [|z| > alpha / 2]; for the percentile
scale, the inverse normal CDF against an independent erfc, the quantile against order
statistics interpolated by hand, sigma_hat of Gaussian tokens against their standard
deviation, and clipping of outliers.
"""
from __future__ import annotations

import numpy as np
from scipy.special import ndtri

EPS = 1e-10
PCT_RHO = 0.9995      # CentriQ Tab. 3: activation quantile
PCT_GAMMA = 2.5591    # CentriQ Tab. 3: clip factor gamma*


def center(x: np.ndarray):
    """(x - mean * 1, mean) with the mean over the native channels of each token."""
    x = np.asarray(x, dtype=np.float64)
    mean = x.sum(axis=1) / x.shape[1]
    return x - mean[:, None], mean


def absmax_quantize(z: np.ndarray, qmax: int, eps: float = EPS):
    """Eq. 1 with r = ||z||_inf: returns (int64 codes [T, d], alpha float64 [T])."""
    z = np.asarray(z, dtype=np.float64)
    r = np.max(np.abs(z), axis=1)
    alpha = np.maximum(r, eps) / qmax
    q = np.clip(np.rint(z / alpha[:, None]), -qmax, qmax).astype(np.int64)
    return q, alpha


def lloyd_max_quantize(z: np.ndarray, thresholds: np.ndarray, eps: float = EPS):
    """Nearest-centroid Lloyd-Max codes of z / sigma: (int64 codes [T, d], sigma [T])."""
    z = np.asarray(z, dtype=np.float64)
    sigma = np.maximum(np.sqrt(np.mean(z * z, axis=1)), eps)
    u = z / sigma[:, None]
    # number of thresholds strictly below u (searchsorted 'left' counts tau_k < u)
    codes = np.searchsorted(np.asarray(thresholds, dtype=np.float64), u, side="left")
    return codes.astype(np.int64), sigma


def percentile_quantize(z: np.ndarray, qmax: int, rho: float = PCT_RHO,
                        gamma: float = PCT_GAMMA, eps: float = EPS):
    """Eq. 1 with the percentile range (CentriQ §4.2, App. B.3): (int64 codes, alpha [T]).

    sigma_hat = q_rho(|z|) / Phi^-1((1 + rho) / 2); alpha = max(gamma sigma_hat, eps) / qmax;
    codes = clip(round(z / alpha), -qmax, qmax).
    """
    z = np.asarray(z, dtype=np.float64)
    q = np.quantile(np.abs(z), rho, axis=1)          # linear between order statistics
    sigma_hat = q / ndtri((1.0 + rho) / 2.0)
    alpha = np.maximum(gamma * sigma_hat, eps) / qmax
    codes = np.clip(np.rint(z / alpha[:, None]), -qmax, qmax).astype(np.int64)
    return codes, alpha


def pack_nibbles(v: np.ndarray) -> np.ndarray:
    """Pack 4-bit values (signed -8..7 or unsigned 0..15) of [R, d] into uint8 [R, d/2]."""
    v = np.asarray(v, dtype=np.int64)
    if v.shape[-1] % 2:
        raise ValueError("even width required")
    n = v & 0xF
    return (n[..., 0::2] | (n[..., 1::2] << 4)).astype(np.uint8)


def pack_pairs(v: np.ndarray) -> np.ndarray:
    """Pack 2-bit signed values (-2..1; the A2 grid uses -1..1) of [R, d] into uint8 [R, d/4]."""
    v = np.asarray(v, dtype=np.int64)
    if v.shape[-1] % 4:
        raise ValueError("width must be a multiple of 4")
    n = v & 0x3
    return (n[..., 0::4] | (n[..., 1::4] << 2) | (n[..., 2::4] << 4)
            | (n[..., 3::4] << 6)).astype(np.uint8)


def unpack_pairs(b: np.ndarray) -> np.ndarray:
    """Inverse of ``pack_pairs``: uint8 [R, d/4] -> int64 [R, d] in -2..1."""
    b = np.asarray(b, dtype=np.int64)
    out = np.empty(b.shape[:-1] + (4 * b.shape[-1],), dtype=np.int64)
    for i in range(4):
        out[..., i::4] = (b >> (2 * i)) & 0x3
    return np.where(out >= 2, out - 4, out)


def unpack_nibbles(b: np.ndarray, signed: bool) -> np.ndarray:
    """Inverse of ``pack_nibbles``: uint8 [R, d/2] -> int64 [R, d]."""
    b = np.asarray(b, dtype=np.int64)
    lo, hi = b & 0xF, (b >> 4) & 0xF
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int64)
    out[..., 0::2], out[..., 1::2] = lo, hi
    if signed:
        out = np.where(out >= 8, out - 16, out)
    return out
