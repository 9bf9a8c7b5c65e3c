"""The rotated, quantized linear layer end to end -- oracle (test infrastructure).

What the pages fix:
- CentriQ §3: a linear layer computes y_t = W x_t + b; the orthogonal rotation folds into
  the weight, W x = (W Q^T)(Q x).
- CentriQ §4.2, Eq. 4: W x_t = W x_t^c + mean_t * w_1 with w_1 = W 1 computed once in FP32
  from the unquantized weight (here in float64).
- CentriQ §4.2, Eq. 5 and App. B.2, Eq. 9: y_t = W_hat Q_a(Q x_t^c) + mean_t * w_1 + b, with
  the rank-1 term and the bias added in the GEMM epilogue.
- W4A2 (CentriQ App. C.1, Tab. 4): the same layer with b = 2 activations (percentile range,
  grid {-1, 0, 1}); the integer GEMM and the epilogue are unchanged.
- Weights: symmetric INT4 per output channel on the pre-rotated weight W_R = W Q^T
  (grid {-7..7}, CentriQ Eq. 1 applied to the rows of W_R; the task fixes per-channel INT4).

Readings: the weight rows are rotated with the activation plan and no centering; the
per-channel scale uses the same eps floor as the activations; the Lloyd-Max dequantised
activation is sigma_t * c[code].

Parity: pinned (tests/test_oracle_linear.py): the integer GEMM against an int64 triple loop;
the rank-1 identity W(x - mean 1) + mean W 1 = W x in float64; with the quantizers replaced by
the identity the layer returns W x + b (CentriQ App. C.5 "Exactness of the re-injection");
offset invariance y(x + c 1) = y(x) + c w_1 (CentriQ Eq. 6).
"""
from __future__ import annotations

import numpy as np

from .quant import EPS, center, absmax_quantize, lloyd_max_quantize, percentile_quantize
from .rpbh import rotate

QMAX = {"int8_absmax": 127, "int4_absmax": 7}


def quantize_activations(x: np.ndarray, plan, h: int, act: str, center_tokens: bool,
                         thresholds: np.ndarray | None = None):
    """Center (optional) -> RPBH rounds -> per-token scale -> codes.

    Returns a dict with ``rotated`` (float64 [T, d], normalised), ``codes`` (int64 [T, d]),
    ``scale`` (alpha or sigma, float64 [T]) and ``mean`` (float64 [T], zeros if not centered).
    """
    x = np.asarray(x, dtype=np.float64)
    if center_tokens:
        xc, mean = center(x)
    else:
        xc, mean = x, np.zeros(x.shape[0])
    z = rotate(xc, plan, h)
    if act in QMAX:
        codes, scale = absmax_quantize(z, QMAX[act])
    elif act in ("int4_lloydmax", "int4_lloydmax_width", "int8_lloydmax"):
        codes, scale = lloyd_max_quantize(z, thresholds)
    elif act == "int4_percentile":
        codes, scale = percentile_quantize(z, 7)
    elif act == "int2_percentile":
        codes, scale = percentile_quantize(z, 1)       # b = 2: grid {-1, 0, 1}
    else:
        raise ValueError(act)
    return {"rotated": z, "codes": codes, "scale": scale, "mean": mean}


def prepare_weights(w: np.ndarray, plan, h: int):
    """W_R = W Q^T (each row rotated), INT4 per output channel, and w_1 = W 1.

    Returns (codes int64 [N, d] in {-7..7}, s_w float64 [N], w_1 float64 [N]).
    """
    w = np.asarray(w, dtype=np.float64)
    w_r = rotate(w, plan, h)
    codes, s_w = absmax_quantize(w_r, 7, EPS)
    w1 = w.sum(axis=1)
    return codes, s_w, w1


def gemm_int(a_codes: np.ndarray, w_codes: np.ndarray) -> np.ndarray:
    """acc[t, o] = sum_k a[t, k] w[o, k], exact: float64 BLAS on integers below 2^53."""
    a = np.asarray(a_codes, dtype=np.float64)
    w = np.asarray(w_codes, dtype=np.float64)
    bound = np.abs(a).max(initial=0) * np.abs(w).max(initial=0) * a.shape[1]
    if bound >= 2.0 ** 53:
        raise ValueError("integer GEMM would not be exact in float64")
    return a @ w.T


def gemm_lloyd_max(codes: np.ndarray, centroids: np.ndarray, w_codes: np.ndarray):
    """acc[t, o] = sum_k c[code[t, k]] w[o, k] in float64."""
    return np.asarray(centroids, dtype=np.float64)[codes] @ np.asarray(w_codes,
                                                                         np.float64).T


def epilogue(acc, scale, s_w, mean=None, w1=None, bias=None):
    """Eq. 5 / Eq. 9: y = scale_t * s_w[o] * acc + mean_t * w_1[o] + b[o] (float64)."""
    y = acc * np.asarray(scale)[:, None] * np.asarray(s_w)[None, :]
    if mean is not None:
        y = y + np.asarray(mean)[:, None] * np.asarray(w1)[None, :]
    if bias is not None:
        y = y + np.asarray(bias)[None, :]
    return y


def linear_forward(x, w, plan, h, act, center_tokens, bias=None, centroids=None,
                   thresholds=None):
    """The whole quantized layer in float64. Returns (y, activation dict, weight tuple)."""
    qa = quantize_activations(x, plan, h, act, center_tokens, thresholds)
    w_codes, s_w, w1 = prepare_weights(w, plan, h)
    if act in ("int4_lloydmax", "int4_lloydmax_width", "int8_lloydmax"):
        acc = gemm_lloyd_max(qa["codes"], centroids, w_codes)
    else:
        acc = gemm_int(qa["codes"], w_codes)
    y = epilogue(acc, qa["scale"], s_w, qa["mean"] if center_tokens else None,
                 w1 if center_tokens else None, bias)
    return y, qa, (w_codes, s_w, w1)


def linear_unquantized(x, w, plan, h, center_tokens, bias=None):
    """Eq. 5 with Q_a = identity and W_hat_R = W Q^T unquantized (CentriQ App. C.5)."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    if center_tokens:
        xc, mean = center(x)
    else:
        xc, mean = x, None
    z = rotate(xc, plan, h)
    w_r = rotate(w, plan, h)
    y = z @ w_r.T
    if mean is not None:
        y = y + mean[:, None] * w.sum(axis=1)[None, :]
    if bias is not None:
        y = y + np.asarray(bias)[None, :]
    return y
