"""Comparison helpers for the parity tests (GPU results against the oracle).

Tolerances (stated for this layer): rotated values <= 1e-5 relative to fp64 (Frobenius,
per token); codes identical except where the oracle value lies within 1e-5 relative of a
decision boundary; integer accumulators bit-exact given the same codes; final bf16 outputs
<= 8e-3 relative (Frobenius over the whole output).
"""
from __future__ import annotations

import numpy as np

ROT_TOL = 1e-5
BOUNDARY_REL = 1e-5
OUT_TOL = 8e-3


def pack_w4_gemm(w) -> np.ndarray:
    """INT4 weight codes [N, K] (-8..7) -> the prepared-weight GEMM layout of include/oq.h:
    every row in 16-byte groups, byte j of group g holding element 32g + j in bits 0-3 and
    element 32g + 16 + j in bits 4-7."""
    w = np.asarray(w, dtype=np.int64)
    n, k = w.shape
    if k % 32:
        raise ValueError("K must be a multiple of 32")
    g = (w & 0xF).reshape(n, k // 32, 32)
    return (g[..., :16] | (g[..., 16:] << 4)).reshape(n, k // 2).astype(np.uint8)


def unpack_w4_gemm(b) -> np.ndarray:
    """Inverse of ``pack_w4_gemm``: uint8 [N, K/2] -> signed int64 [N, K]."""
    b = np.asarray(b, dtype=np.int64)
    n, kb = b.shape
    g = b.reshape(n, kb // 16, 16)
    out = np.concatenate([g & 0xF, (g >> 4) & 0xF], axis=-1).reshape(n, kb * 2)
    return np.where(out >= 8, out - 16, out)


def to_torch_bf16(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).to(device)


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a - b))


def per_token_rel(a, b) -> np.ndarray:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b, axis=1)
    return np.linalg.norm(a - b, axis=1) / np.where(nb > 0, nb, 1.0)


def absmax_boundary_mask(z: np.ndarray, alpha: np.ndarray, qmax: int) -> np.ndarray:
    """True where z / alpha lies within 1e-5 relative of a rounding boundary k + 1/2
    (or of the clip edge qmax, whose neighbourhood both sides round identically)."""
    v = z / alpha[:, None]
    k = np.floor(v)
    b = k + 0.5
    near = np.abs(v - b) <= BOUNDARY_REL * np.maximum(np.abs(b), 0.5)
    return near & (np.abs(b) < qmax)


def lloyd_max_boundary_mask(z: np.ndarray, sigma: np.ndarray, thresholds) -> np.ndarray:
    u = z / sigma[:, None]
    t = np.asarray(thresholds, dtype=np.float64)
    d = np.abs(u[..., None] - t[None, None, :])
    return np.any(d <= BOUNDARY_REL * np.maximum(np.abs(t), 1.0)[None, None, :], axis=-1)


def compare_codes(gpu_codes: np.ndarray, ref_codes: np.ndarray, exempt: np.ndarray):
    """(number of differing codes outside the exemption, number of exempted positions)."""
    diff = gpu_codes != ref_codes
    return int(np.sum(diff & ~exempt)), int(np.sum(exempt))


def fp16_boundary_mask(x: np.ndarray, floor: float = 0.0) -> np.ndarray:
    """True where float64 x lies within 1e-5 * max(|x|, floor) of a rounding boundary of
    fp16 (the midpoint between two neighbouring fp16 values), so that a computation that
    reaches x with a relative error below 1e-5 may round it to either neighbour."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float16)
    up = np.nextafter(f, np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(f, np.float16(-np.inf)).astype(np.float64)
    fd = f.astype(np.float64)
    gap = np.minimum(np.abs(x - (fd + up) / 2), np.abs(x - (fd + dn) / 2))
    return gap <= BOUNDARY_REL * np.maximum(np.abs(x), floor)


def grid_boundary_mask(v: np.ndarray, lo: int, hi: int) -> np.ndarray:
    """True where v lies within 1e-5 relative (floor 1/2) of a rounding boundary k + 1/2 with
    lo <= k < hi, i.e. where round-half-even to the integers in [lo, hi] is decided by noise."""
    v = np.asarray(v, dtype=np.float64)
    b = np.floor(v) + 0.5
    near = np.abs(v - b) <= BOUNDARY_REL * np.maximum(np.abs(b), 0.5)
    return near & (b > lo) & (b < hi)
