"""Pins for the oracle's whole layer (CPU only).

CentriQ §3 (y = W x + b, rotation folded into the weight), §4.2 Eq. 4 (rank-1 identity),
Eq. 5 / App. B.2 Eq. 9 (forward pass), Eq. 6 (offset invariance), App. C.5 (identity
quantizer recovers W x + b exactly).
"""
import numpy as np
import pytest

import oracle
import synth
from oracle import linear as Lm


def brute_gemm(a, w):
    T, K = a.shape
    N = w.shape[0]
    out = np.zeros((T, N), dtype=np.int64)
    for t in range(T):
        for o in range(N):
            s = 0
            for k in range(K):
                s += int(a[t, k]) * int(w[o, k])
            out[t, o] = s
    return out


def check_gemm():
    rng = np.random.default_rng(7)
    a = rng.integers(-127, 128, (5, 37))
    w = rng.integers(-7, 8, (6, 37))
    return bool(np.array_equal(Lm.gemm_int(a, w), brute_gemm(a, w).astype(np.float64)))


def check_identity_quantizer(center, rounds, bias):
    rng = np.random.default_rng(8)
    d, n, h = 256, 48, 64
    x = rng.standard_normal((6, d)) + rng.standard_normal((6, 1)) * 3
    w = rng.standard_normal((n, d)) / np.sqrt(d)
    b = rng.standard_normal(n) if bias else None
    plan = oracle.rpbh_plan(d, h, rounds, 0)
    y = Lm.linear_unquantized(x, w, plan, h, center, b)
    ref = x @ w.T + (0 if b is None else b[None, :])
    return float(np.abs(y - ref).max() / np.abs(ref).max()) < 1e-12


def check_lm_gemm():
    rng = np.random.default_rng(9)
    c, _ = oracle.lloyd_max_gaussian()
    codes = rng.integers(0, 16, (4, 33))
    w = rng.integers(-7, 8, (5, 33))
    want = np.array([[sum(c[codes[t, k]] * w[o, k] for k in range(33)) for o in range(5)]
                     for t in range(4)])
    return float(np.abs(Lm.gemm_lloyd_max(codes, c, w) - want).max()) < 1e-12


def test_integer_gemm_is_exact():
    assert check_gemm()


def test_lloyd_max_gemm_matches_loop():
    assert check_lm_gemm()


def test_rank1_identity_eq4():
    rng = np.random.default_rng(10)
    x = rng.standard_normal((7, 192)) + 5.0
    w = rng.standard_normal((33, 192))
    xc, mean = oracle.center(x)
    lhs = xc @ w.T + mean[:, None] * w.sum(axis=1)[None, :]
    assert np.abs(lhs - x @ w.T).max() < 1e-12 * np.abs(x @ w.T).max()


@pytest.mark.parametrize("center,rounds,bias", [(False, 1, False), (True, 1, True),
                                                (True, 2, False), (False, 2, True)])
def test_identity_quantizer_recovers_wx_plus_b(center, rounds, bias):
    assert check_identity_quantizer(center, rounds, bias)


def test_prepare_weights_definition():
    rng = np.random.default_rng(12)
    d, n, h = 128, 16, 32
    w = rng.standard_normal((n, d))
    plan = oracle.rpbh_plan(d, h, 2, 0)
    codes, s_w, w1 = oracle.prepare_weights(w, plan, h)
    w_r = oracle.rotate(w, plan, h)
    assert np.allclose(w1, w.sum(axis=1), rtol=0, atol=1e-12)
    assert np.allclose(s_w, np.abs(w_r).max(axis=1) / 7, rtol=1e-15)
    assert np.all(np.abs(codes) <= 7)
    assert np.abs(codes * s_w[:, None] - w_r).max() <= 0.5 * s_w.max() * (1 + 1e-12)


def test_offset_invariance_of_quantized_layer_eq6():
    rng = np.random.default_rng(13)
    d, n, h = 256, 32, 64
    x = np.round(rng.standard_normal((6, d)) * 16) / 16
    w = rng.standard_normal((n, d)) / np.sqrt(d)
    plan = oracle.rpbh_plan(d, h, 1, 0)
    c = 0.375
    y1, qa1, (_, _, w1) = oracle.linear_forward(x, w, plan, h, "int4_absmax", True)
    y2, qa2, _ = oracle.linear_forward(x + c, w, plan, h, "int4_absmax", True)
    assert np.array_equal(qa1["codes"], qa2["codes"])
    assert np.array_equal(qa1["scale"], qa2["scale"])
    assert np.abs(y2 - (y1 + c * w1[None, :])).max() < 1e-12 * np.abs(y2).max()


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_quantized_layer_tracks_full_precision():
    # diagnostic, not parity: the layer's error against W x stays in the range expected
    # of INT4 weights with A8 / A4 activations.
    wl, xb, wb = synth.make_inputs("tiny")
    x, w = synth.bf16_to_f64(xb), synth.bf16_to_f64(wb)
    plan = oracle.rpbh_plan(wl.d, wl.h, wl.rounds, 0)
    y, _, _ = oracle.linear_forward(x, w, plan, wl.h, "int8_absmax", False)
    assert _rel(y, x @ w.T) < 0.15


def test_centering_lowers_error_with_large_token_means():
    # CentriQ §4.1-4.2: with a large per-token mean, centering before rotation lowers
    # the A4 quantisation error (the mean no longer sets the per-token range).
    wl = synth.WORKLOADS["mlp_up"]
    xb = synth.make_x(64, 512, mean_var=25.0, seed=1)
    wb = synth.make_w(64, 512, seed=1)
    x, w = synth.bf16_to_f64(xb), synth.bf16_to_f64(wb)
    h = 512
    plan = oracle.rpbh_plan(512, h, 1, 0)
    ref = x @ w.T
    # isolate the activation quantiser: full-precision rotated weights
    def act_only(center):
        qa = oracle.quantize_activations(x, plan, h, "int4_absmax", center)
        deq = qa["codes"] * qa["scale"][:, None]
        w_r = oracle.rotate(w, plan, h)
        return deq @ w_r.T + (qa["mean"][:, None] * w.sum(axis=1)[None, :] if center else 0)
    e_plain, e_center = _rel(act_only(False), ref), _rel(act_only(True), ref)
    assert e_center < e_plain
    assert wl.center
