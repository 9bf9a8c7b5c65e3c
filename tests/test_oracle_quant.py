"""Pins for the oracle's centering, quantizers and nibble packing (CPU only).

CentriQ §3 Eq. 1 (symmetric per-token grid), §4.2 (centering; "Scale and grid": the
percentile scale), Eq. 6 (offset invariance), App. B.3 Tab. 3 (rho, gamma*);
OrbitQuant PR #25 (absmax A8, Lloyd-Max below 8 bits).
"""
import math

import numpy as np
import pytest

import oracle
from oracle import quant as Qm


def check_absmax(z, qmax):
    q, alpha = Qm.absmax_quantize(z, qmax)
    ok = True
    # the largest coordinate lands on the end of the grid
    j = np.argmax(np.abs(z), axis=1)
    ok &= bool(np.all(np.abs(q[np.arange(len(z)), j]) == qmax))
    # rounding error at most half a step, codes inside the grid
    ok &= bool(np.all(np.abs(z - alpha[:, None] * q) <= alpha[:, None] * (0.5 + 1e-12)))
    ok &= bool(np.all(np.abs(q) <= qmax))
    # brute force: nearest grid point
    grid = np.arange(-qmax, qmax + 1)
    dist = np.abs(z[..., None] - alpha[:, None, None] * grid[None, None, :])
    best = grid[np.argmin(dist, axis=-1)]
    tie = np.sort(dist, axis=-1)
    clear = (tie[..., 1] - tie[..., 0]) > 1e-12 * alpha[:, None]
    ok &= bool(np.all(best[clear] == q[clear]))
    return ok


def check_lloyd_max_codes(z):
    c, t = oracle.lloyd_max_gaussian()
    codes, sigma = Qm.lloyd_max_quantize(z, t)
    u = z / sigma[:, None]
    dist = np.abs(u[..., None] - c[None, None, :])
    srt = np.sort(dist, axis=-1)
    clear = (srt[..., 1] - srt[..., 0]) > 1e-12
    ok = bool(np.all(np.argmin(dist, axis=-1)[clear] == codes[clear]))
    ok &= bool(np.allclose(sigma, np.sqrt((z * z).mean(axis=1)), rtol=1e-14))
    return ok


@pytest.mark.parametrize("qmax", [127, 7])
def test_absmax_quantizer(qmax):
    rng = np.random.default_rng(1)
    z = rng.standard_normal((40, 96)) * rng.uniform(0.01, 100, (40, 1))
    assert check_absmax(z, qmax)


def test_absmax_zero_row_uses_eps():
    q, alpha = Qm.absmax_quantize(np.zeros((2, 16)), 127)
    assert np.all(q == 0) and np.allclose(alpha, 1e-10 / 127)


def test_lloyd_max_codes_are_nearest_centroid():
    rng = np.random.default_rng(2)
    z = rng.standard_normal((30, 128)) * rng.uniform(0.1, 5, (30, 1))
    assert check_lloyd_max_codes(z)


def test_lloyd_max_threshold_tie_goes_low():
    c, t = oracle.lloyd_max_gaussian()
    # a token whose RMS is exactly 1 and that holds values exactly on thresholds
    z = np.array([[t[3], -t[3], t[10], -t[10]]])
    z = z / np.sqrt(np.mean(z * z))
    codes, sigma = Qm.lloyd_max_quantize(z, t)
    u = z / sigma[:, None]
    assert np.all(codes == np.searchsorted(t, u[0], side="left"))


def test_centering_and_offset_invariance():
    # CentriQ Eq. 6: codes and scale of the centered token do not depend on x + c 1.
    # x on a 2^-4 grid and c = 3/8 keep every sum exact in float64.
    rng = np.random.default_rng(3)
    x = np.round(rng.standard_normal((8, 256)) * 16) / 16
    c = 3.0 / 8.0
    xc1, m1 = Qm.center(x)
    xc2, m2 = Qm.center(x + c)
    assert np.array_equal(xc1, xc2) and np.array_equal(m2 - m1, np.full(8, c))
    assert np.allclose(xc1.sum(axis=1), 0.0, atol=1e-12)
    plan = oracle.rpbh_plan(256, 64, 1, 0)
    z1 = oracle.rotate(xc1, plan, 64)
    z2 = oracle.rotate(xc2, plan, 64)
    q1, a1 = Qm.absmax_quantize(z1, 7)
    q2, a2 = Qm.absmax_quantize(z2, 7)
    assert np.array_equal(q1, q2) and np.array_equal(a1, a2)


def test_pack_nibbles_hand_examples():
    assert Qm.pack_nibbles(np.array([[1, -1]]))[0, 0] == 0xF1
    assert Qm.pack_nibbles(np.array([[-7, 7]]))[0, 0] == 0x79
    assert Qm.pack_nibbles(np.array([[0, 15]]))[0, 0] == 0xF0
    assert Qm.pack_nibbles(np.array([[3, 0, -8, 2]])).tolist() == [[0x03, 0x28]]


def test_pack_unpack_round_trip():
    rng = np.random.default_rng(4)
    s = rng.integers(-7, 8, (5, 64))
    assert np.array_equal(Qm.unpack_nibbles(Qm.pack_nibbles(s), signed=True), s)
    u = rng.integers(0, 16, (5, 64))
    assert np.array_equal(Qm.unpack_nibbles(Qm.pack_nibbles(u), signed=False), u)


def half_normal_quantile(p):
    """x with Phi(x) = p, by bisection on Phi(x) = erfc(-x / sqrt 2) / 2 (no SciPy)."""
    lo, hi = 0.0, 20.0
    for _ in range(200):
        mid = (lo + hi) / 2
        if 0.5 * math.erfc(-mid / math.sqrt(2.0)) < p:
            lo = mid
        else:
            hi = mid
    return (lo + hi) / 2


def check_percentile(z, qmax=7):
    """The percentile quantizer against its definition written out by hand."""
    q, alpha = Qm.percentile_quantize(z, qmax)
    n = z.shape[1]
    s = np.sort(np.abs(z), axis=1)
    pos = Qm.PCT_RHO * (n - 1)
    k = int(math.floor(pos))
    qv = s[:, k] + (pos - k) * (s[:, min(k + 1, n - 1)] - s[:, k])
    sigma_hat = qv / half_normal_quantile((1 + Qm.PCT_RHO) / 2)
    alpha_ref = np.maximum(Qm.PCT_GAMMA * sigma_hat, Qm.EPS) / qmax
    ok = bool(np.allclose(alpha, alpha_ref, rtol=1e-12, atol=0))
    # codes: the nearest point of the grid {-qmax..qmax} (values past the range clip)
    grid = np.arange(-qmax, qmax + 1)
    dist = np.abs(z[..., None] - alpha[:, None, None] * grid[None, None, :])
    best = grid[np.argmin(dist, axis=-1)]
    tie = np.sort(dist, axis=-1)
    clear = (tie[..., 1] - tie[..., 0]) > 1e-12 * alpha[:, None]
    ok &= bool(np.all(best[clear] == q[clear]))
    return ok


def test_half_normal_quantile_pin():
    # the table value of the standard normal 0.99975 quantile, and SciPy agrees with erfc
    x = half_normal_quantile(0.99975)
    assert abs(x - 3.4807564) < 1e-6
    assert abs(Qm.ndtri(0.99975) - x) < 1e-12


@pytest.mark.parametrize("n", [256, 1920, 3072, 4096, 30720])
def test_percentile_quantizer_definition(n):
    z = np.random.default_rng(n).standard_normal((6, n)) * np.array([[0.5], [1], [2], [3], [7], [1e-3]])
    assert check_percentile(z)


def test_percentile_scale_of_gaussian_tokens():
    # sigma_hat estimates the standard deviation of a Gaussian token (the Phi^-1 normalisation)
    rng = np.random.default_rng(3)
    for sd in (0.1, 1.0, 5.0):
        z = rng.normal(0, sd, (2, 400000))
        _, alpha = Qm.percentile_quantize(z, 7)
        sigma_hat = alpha * 7 / Qm.PCT_GAMMA
        assert np.all(np.abs(sigma_hat / sd - 1) < 0.04)


def test_percentile_clips_outliers():
    # one huge coordinate moves the quantile by at most one rank of the clean magnitudes (unlike
    # an absmax range, which it would set) and clips to the end of the grid
    n = 4096
    z = np.random.default_rng(4).standard_normal((1, n))
    s = np.sort(np.abs(z[0]))
    k = int(math.floor(Qm.PCT_RHO * (n - 1)))
    z[0, 17] = 1000.0
    q, a1 = Qm.percentile_quantize(z, 7)
    quantile = a1[0] * 7 / Qm.PCT_GAMMA * half_normal_quantile((1 + Qm.PCT_RHO) / 2)
    assert s[k] <= quantile <= s[k + 2]
    assert q[0, 17] == 7
    assert q.min() >= -7 and q.max() <= 7


# ---- A2: the b = 2 grid of CentriQ Eq. 1 (W4A2, App. C.1 Tab. 4; Tab. 3 scale) ----------------

def check_pairs():
    """2-bit packing: hand-written bytes and a round trip."""
    v = np.array([[1, 0, -1, 0, -1, -1, -1, -1, 0, 1, 0, 1]])
    b = [[0b00110001, 0xFF, 0b01000100]]
    ok = Qm.pack_pairs(v).tolist() == b
    ok &= Qm.unpack_pairs(np.array(b, np.uint8)).tolist() == v.tolist()
    s = np.random.default_rng(5).integers(-1, 2, (5, 64))
    ok &= bool(np.array_equal(Qm.unpack_pairs(Qm.pack_pairs(s)), s))
    return ok


def check_ternary(z):
    """qmax = 1: the nearest point of {-1, 0, 1} is sign(z) where |z| > alpha / 2, else 0
    (round half to even sends |z| = alpha / 2 to 0), and alpha is gamma sigma_hat itself."""
    q, alpha = Qm.percentile_quantize(z, 1)
    _, alpha7 = Qm.percentile_quantize(z, 7)
    ref = np.where(np.abs(z) > alpha[:, None] / 2, np.sign(z), 0).astype(np.int64)
    return bool(np.allclose(alpha, 7 * alpha7, rtol=1e-15) and np.array_equal(q, ref))


def check_layer_a2():
    """The layer oracle's A2 kind: percentile codes on the grid {-1, 0, 1}."""
    from oracle import linear as L, rpbh_plan
    x = np.random.default_rng(9).standard_normal((3, 256)) + 2.0
    qa = L.quantize_activations(x, rpbh_plan(256, 64, 1, 0), 64, "int2_percentile", True)
    q, a = Qm.percentile_quantize(qa["rotated"], 1)
    return bool(set(np.unique(qa["codes"])) <= {-1, 0, 1} and np.array_equal(q, qa["codes"])
                and np.allclose(a, qa["scale"], rtol=0))


def test_pack_pairs():
    # element 4j + i in bits 2i, 2i + 1 of byte j, two's complement (-1 = 0b11)
    assert check_pairs()
    with pytest.raises(ValueError):
        Qm.pack_pairs(np.zeros((1, 6), np.int64))


@pytest.mark.parametrize("n", [256, 3072])
def test_ternary_percentile_definition(n):
    # qmax = 1: the same quantile and clip (Tab. 3 is one setting for every b), grid {-1, 0, 1}
    z = np.random.default_rng(n + 1).standard_normal((5, n)) * np.array([[0.5], [1], [3], [7], [1e-3]])
    assert check_percentile(z, qmax=1)


def test_ternary_codes_closed_form():
    rng = np.random.default_rng(8)
    assert check_ternary(rng.standard_normal((4, 1024)) * 2.0)
    # exact half steps go to 0, and anything past 1.5 alpha clips to +-1: two of the smallest
    # magnitudes become +-alpha / 2 and one becomes an outlier; alpha / 2 lies far below the
    # quantile's order statistics, so alpha only moves with the outlier (by one rank)
    z2 = rng.standard_normal((1, 4000))
    small = np.argsort(np.abs(z2[0]))[:3]
    z2[0, small[2]] = 1e3
    _, a = Qm.percentile_quantize(z2, 1)
    z2[0, small[0]], z2[0, small[1]] = a[0] / 2, -a[0] / 2
    q2, a2 = Qm.percentile_quantize(z2, 1)
    assert a2[0] == a[0]
    assert q2[0, small[0]] == 0 and q2[0, small[1]] == 0 and q2[0, small[2]] == 1


def test_layer_oracle_accepts_a2():
    assert check_layer_a2()
