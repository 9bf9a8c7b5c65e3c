"""Pins for the oracle's 16-level N(0,1) Lloyd-Max codebook (CPU only).

The optimality conditions are the definition of a Lloyd-Max quantizer; Max (1960) tabulates
the 16-level Gaussian quantizer; scipy.optimize minimises the distortion by a different
method (Nelder-Mead on the thresholds). OrbitQuant PR #25 "Default changes" names the
codebook and its solvers.
"""
import os

import numpy as np
from scipy.optimize import minimize
from scipy.special import ndtr

import oracle
from oracle import lloyd_max as L


def _phi(x):
    return np.exp(-0.5 * x * x) / np.sqrt(2 * np.pi)


def check_conditions(c, t):
    edges = np.concatenate(([-np.inf], t, [np.inf]))
    p = ndtr(edges[1:]) - ndtr(edges[:-1])
    phi = np.where(np.isfinite(edges), _phi(np.where(np.isfinite(edges), edges, 0.0)), 0.0)
    with np.errstate(invalid="ignore", divide="ignore"):
        cond_centroid = np.nanmax(np.abs(c - (phi[:-1] - phi[1:]) / p))
    cond_mid = np.abs(t - 0.5 * (c[:-1] + c[1:])).max()
    return cond_centroid < 1e-12 and cond_mid < 1e-15


def load_max1960(golden_dir):
    rows = [l.split() for l in open(os.path.join(golden_dir,
                                                 "lloyd_max_16_gaussian_max1960.txt"))
            if l.strip() and not l.startswith("#")]
    return rows


def check_max1960(c, t, golden_dir):
    ok = True
    for kind, idx, val in load_max1960(golden_dir):
        got = (t if kind == "threshold" else c)[int(idx)]
        ok &= abs(got - float(val)) <= 6e-4
    return ok


def test_optimality_conditions():
    c, t = oracle.lloyd_max_gaussian()
    assert check_conditions(c, t)


def test_odd_symmetry():
    c, t = oracle.lloyd_max_gaussian()
    assert np.abs(c + c[::-1]).max() < 1e-13
    assert np.abs(t + t[::-1]).max() < 1e-13
    assert np.all(np.diff(c) > 0) and np.all(np.diff(t) > 0)


def test_matches_max_1960_table(golden_dir):
    c, t = oracle.lloyd_max_gaussian()
    assert check_max1960(c, t, golden_dir)


def test_agrees_with_direct_minimisation():
    c, t = oracle.lloyd_max_gaussian()

    def distortion(pos):
        tt = np.sort(np.concatenate((-pos[::-1], [0.0], pos)))
        e = np.concatenate(([-np.inf], tt, [np.inf]))
        p = L._cell_prob(e[:-1], e[1:])
        cc = (L._phi(e[:-1]) - L._phi(e[1:])) / p
        return L.lloyd_max_mse(cc, tt)

    r = minimize(distortion, t[8:] + 0.05, method="Nelder-Mead",
                 options=dict(xatol=1e-12, fatol=1e-17, maxiter=50000, maxfev=100000))
    assert np.abs(np.sort(r.x) - t[8:]).max() < 1e-6
    assert abs(r.fun - L.lloyd_max_mse(c, t)) < 1e-13


def test_mse_closed_form_matches_monte_carlo():
    c, t = oracle.lloyd_max_gaussian()
    x = np.random.default_rng(5).standard_normal(2_000_000)
    q = c[np.searchsorted(t, x)]
    mc = float(np.mean((x - q) ** 2))
    assert abs(mc - L.lloyd_max_mse(c, t)) < 3e-4 * 1.0
    assert 0.0094 < L.lloyd_max_mse(c, t) < 0.0096


# ---- per-width tables: the width-d post-rotation marginal f_d -----------------------------

def test_sphere_d3_is_the_uniform_quantizer():
    # f_3 is uniform on [-sqrt 3, sqrt 3]: the Lloyd-Max quantizer of a uniform density has
    # equal cells, centroids at the cell midpoints (closed form)
    d, L16 = 3, 16
    c, t = oracle.lloyd_max_sphere(d)
    r = np.sqrt(3.0)
    edges = -r + 2 * r * np.arange(L16 + 1) / L16
    assert np.allclose(t, edges[1:-1], atol=1e-12)
    assert np.allclose(c, 0.5 * (edges[:-1] + edges[1:]), atol=1e-12)


def test_sphere_conditions_by_quadrature():
    # centroid and midpoint conditions, with the cell integrals of f_d done by adaptive
    # quadrature of the density itself (not the incomplete-beta / closed-form pair)
    from scipy.integrate import quad
    for d in (32, 256, 1920):
        pdf, _, _ = oracle.sphere_marginal(d)
        f = lambda y: float(pdf(np.array([y]))[0])
        c, t = oracle.lloyd_max_sphere(d)
        r = min(np.sqrt(d), 12.0)      # f_d < 1e-30 beyond 12 for these widths
        edges = np.concatenate(([-r], t, [r]))
        total = 0.0
        for k in range(16):
            a, b = edges[k], edges[k + 1]
            p = quad(f, a, b, epsabs=1e-14, epsrel=1e-13, limit=200)[0]
            mom = quad(lambda y: y * f(y), a, b, epsabs=1e-14, epsrel=1e-13, limit=200)[0]
            total += p
            assert abs(mom / p - c[k]) < 1e-9, (d, k)
        assert abs(total - 1.0) < 1e-10
        assert np.abs(t - 0.5 * (c[:-1] + c[1:])).max() < 1e-15
        assert np.allclose(c, -c[::-1], atol=1e-12)


def test_sphere_tables_tend_to_the_gaussian_table():
    # the gap to the N(0, 1) table closes like 1/d
    cg, tg = oracle.lloyd_max_gaussian()
    scaled = []
    for d in (1024, 16384, 262144):
        c, _ = oracle.lloyd_max_sphere(d)
        scaled.append(np.abs(c - cg).max() * d)
    assert max(scaled) / min(scaled) < 1.01
    assert scaled[-1] / 262144 < 3e-5


def test_sphere_distortion_monte_carlo():
    # quantize sqrt(d) u_1 for random directions u: the empirical MSE matches the table's
    # distortion computed by quadrature, and beats the Gaussian table on the same samples
    from scipy.integrate import quad
    d = 64
    c, t = oracle.lloyd_max_sphere(d)
    pdf, _, _ = oracle.sphere_marginal(d)
    r = np.sqrt(d)
    edges = np.concatenate(([-r], t, [r]))
    mse = sum(quad(lambda y: (y - c[k]) ** 2 * float(pdf(np.array([y]))[0]), edges[k],
                   edges[k + 1], epsabs=1e-14, limit=200)[0] for k in range(16))
    rng = np.random.default_rng(7)
    u = rng.standard_normal((200000, d))
    y = np.sqrt(d) * u[:, 0] / np.linalg.norm(u, axis=1)
    q = c[np.searchsorted(t, y)]
    emp = np.mean((y - q) ** 2)
    assert abs(emp - mse) < 4e-4 * 3
    cg, tg = oracle.lloyd_max_gaussian()
    assert emp < np.mean((y - cg[np.searchsorted(tg, y)]) ** 2)


# ---- 256 levels: the A8 Lloyd-Max codebook -----------------------------------------------

def test_gaussian_256_levels():
    from scipy.integrate import quad
    c, t = oracle.lloyd_max_gaussian_8bit()
    assert c.shape == (256,) and t.shape == (255,)
    assert np.all(np.diff(c) > 0) and np.allclose(c, -c[::-1], atol=1e-12)
    assert np.abs(t - 0.5 * (c[:-1] + c[1:])).max() < 1e-15
    # centroid condition on sample cells by adaptive quadrature (not the closed form)
    edges = np.concatenate(([-12.0], t, [12.0]))
    for k in (0, 40, 127, 128, 200, 255):
        a, b = edges[k], edges[k + 1]
        p = quad(_phi, a, b, epsabs=1e-16, epsrel=1e-13)[0]
        m = quad(lambda x: x * _phi(x), a, b, epsabs=1e-16, epsrel=1e-13)[0]
        assert abs(m / p - c[k]) < 1e-9 * max(1.0, abs(c[k])), k
    # Panter and Dite (1951): high-resolution distortion sqrt(3) pi / (2 L^2) for N(0, 1)
    mse = L.lloyd_max_mse(c, t)
    assert abs(mse / (np.sqrt(3.0) * np.pi / 2.0 / 256 ** 2) - 1.0) < 0.02
    # Monte Carlo distortion
    x = np.random.default_rng(3).standard_normal(2_000_000)
    emp = np.mean((x - c[np.searchsorted(t, x)]) ** 2)
    assert abs(emp / mse - 1.0) < 0.04   # tail cells dominate the sampling error
