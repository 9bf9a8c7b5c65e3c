"""Pins for the oracle's asymmetric grouped INT4 weights (CentriQ Eq. 2, §4.3, App. B.2)."""
import itertools

import numpy as np

from oracle import weights_g64 as G


def _w(n=6, d=256, seed=0):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((n, d))
    w[0, :64] += 3.0                    # a shifted group
    w[1, 64:128] *= 0.01                # a narrow group
    w[2, 128:192] = 0.25                # a constant group
    return w


def test_reconstruction_error_and_extremes():
    w = _w()
    q, s, z = G.asym_group_quantize(w)
    assert q.min() >= 0 and q.max() <= 15
    wh = G.dequantize(q, s, z)
    err = np.abs(w - wh).reshape(6, 4, 64)
    assert np.all(err <= s[..., None] / 2 * (1 + 1e-12) + 1e-15)
    wg = w.reshape(6, 4, 64)
    whg = wh.reshape(6, 4, 64)
    # the minimum and maximum of every group reconstruct exactly (up to rounding)
    i_lo, i_hi = wg.argmin(axis=2), wg.argmax(axis=2)
    for r, g in itertools.product(range(6), range(4)):
        assert abs(whg[r, g, i_lo[r, g]] - wg[r, g, i_lo[r, g]]) <= 1e-12 * (1 + abs(wg[r, g].max()))
        if wg[r, g].max() > wg[r, g].min():
            assert abs(whg[r, g, i_hi[r, g]] - wg[r, g, i_hi[r, g]]) <= 1e-12 * (1 + abs(wg[r, g].max()))
    # a constant group reconstructs exactly
    assert np.allclose(wh[2, 128:192], 0.25, atol=1e-15)


def test_codes_are_the_nearest_grid_point():
    rng = np.random.default_rng(3)
    w = rng.uniform(-2, 2, (5, 64))
    q, s, z = G.asym_group_quantize(w)
    for r in range(5):
        grid = s[r, 0] * (np.arange(16) - z[r, 0])
        best = np.abs(w[r][:, None] - grid[None, :]).argmin(axis=1)
        d_best = np.abs(w[r] - grid[best])
        d_q = np.abs(w[r] - grid[q[r]])
        assert np.all(d_q <= d_best + 1e-12)


def test_zero_point_correction_identity():
    # App. B.2: the Q - 8 integer product with the correction -sigma z' p equals the product
    # with the dequantized weights
    rng = np.random.default_rng(5)
    w = _w(n=7, d=192, seed=2)
    q, s, z = G.asym_group_quantize(w)
    a = rng.integers(-7, 8, (9, 192))
    ref = a.astype(np.float64) @ G.dequantize(q, s, z).T
    got = G.corrected_product(a, q, s, z)
    assert np.abs(got - ref).max() <= 1e-10 * np.abs(ref).max()


def test_mutation_dropped_correction_is_caught():
    rng = np.random.default_rng(6)
    w = _w(n=4, d=128, seed=4)
    q, s, z = G.asym_group_quantize(w)
    a = rng.integers(-7, 8, (5, 128))
    ref = a.astype(np.float64) @ G.dequantize(q, s, z).T
    ag = a.reshape(5, 2, 64).astype(np.float64)
    qs = (q.astype(np.float64) - 8).reshape(4, 2, 64)
    no_corr = np.einsum("tgk,ngk,ng->tn", ag, qs, s)   # plants the slip: no z' p term
    assert np.abs(no_corr - ref).max() > 1e-3 * np.abs(ref).max()


def test_fp16_storage_codes_nearest_on_stored_grid():
    # with 16-bit storage the codes are the nearest point of the grid that is decoded
    rng = np.random.default_rng(8)
    w = rng.standard_normal((7, 128)) * 0.03
    w[3, :64] += 0.2                       # a group away from zero (negative shift)
    w[4, 64:] *= 1e-3                      # a group below the sigma floor
    q, s, z = G.asym_group_quantize(w, store=np.float16)
    assert np.array_equal(s.astype(np.float16).astype(np.float64), s)
    assert np.array_equal(z.astype(np.float16).astype(np.float64), z)
    assert s.min() >= G.SIGMA_MIN_F16
    for r in range(7):
        for g in range(2):
            grid = s[r, g] * (np.arange(16) - z[r, g])
            seg = w[r, 64 * g:64 * (g + 1)]
            d_best = np.abs(seg[:, None] - grid[None, :]).min(axis=1)
            d_q = np.abs(seg - grid[q[r, 64 * g:64 * (g + 1)]])
            assert np.all(d_q <= d_best + 1e-12)
            # and the stored grid still covers the group (error within one step)
            assert np.all(d_q <= s[r, g] * (0.5 + 2.0 ** -11 * max(1.0, abs(z[r, g]))) + 1e-15)


def test_layer_reduces_to_unquantized_for_fine_weights():
    # the layer oracle with g64 weights, against the unquantized layer: the weight error is
    # bounded by sigma / 2 per element, so |y - y_exact| <= alpha sum_k |a_k| sigma_k / 2 +
    # the activation rounding; checked with the activation quantizer error removed by using
    # the codes' own dequantized activations as input to the exact path
    from oracle import rpbh_plan, rotate
    rng = np.random.default_rng(9)
    d, n, t = 256, 16, 5
    plan = rpbh_plan(d, 64, 1, 0)
    x = rng.standard_normal((t, d))
    w = rng.standard_normal((n, d)) * 0.05
    y, qa, (q, s, z, w1) = G.linear_forward_g64(x, w, plan, 64, "int4_absmax", True)
    a = qa["codes"] * qa["scale"][:, None]                # dequantized activations
    w_r = rotate(w, plan, 64)
    y_exact = a @ w_r.T + qa["mean"][:, None] * w1[None, :]
    sig = np.repeat(s, 64, axis=1)                        # [n, d]
    bound = np.abs(a) @ (sig / 2 + 1e-15).T
    assert np.all(np.abs(y - y_exact) <= bound * (1 + 1e-9))
    assert np.abs(y - y_exact).max() > 0                  # the weights really are quantized


def test_fp16_storage_keeps_the_shift_finite_for_constant_groups():
    # a constant group c has range 0: sigma would be the 2^-14 floor and z = -c 2^14, past the
    # fp16 maximum 65504 once |c| > 4; the |min| / 2^15 floor keeps z finite and the group still
    # reconstructs to within half a grid step (below 2^-15 |c| where that floor is active)
    for c in (5.0, -7.25, 300.0, -0.001, 4.0):
        w = np.full((1, 64), c)
        w[0, 5] = c * (1 + 2.0 ** -20)          # a range far below the floor
        q, s, z = G.asym_group_quantize(w, store=np.float16)
        assert np.all(np.isfinite(z)) and np.abs(z).max() <= 65504
        assert np.array_equal(z.astype(np.float16).astype(np.float64), z)
        assert s[0, 0] >= abs(c) / G.SHIFT_MAX * (1 - 2.0 ** -11)
        err = np.abs(G.dequantize(q, s, z) - w)
        assert err.max() <= s[0, 0] * (0.5 + 2.0 ** -11 * max(1.0, abs(z[0, 0]))) + 1e-300
        if abs(c) >= 2.0:                       # the |min| / 2^15 floor is the active one
            assert err.max() <= abs(c) * 2.0 ** -15
    # a group whose minimum is far from zero with a normal range keeps sigma = range / 15
    w = np.linspace(100.0, 100.5, 64)[None, :]
    q, s, z = G.asym_group_quantize(w, store=np.float16)
    assert s[0, 0] == np.float16(0.5 / 15) and abs(z[0, 0]) < 65504
