"""Planted mistakes in the oracle must be caught by its pins (CPU only).

Each case swaps one oracle function for a copy with a plausible slip (a dropped term, a
wrong sign or index, a transposed operand) and asserts that at least one pin of the
matching test module now fails. Mistakes are planted only in the oracle, on the CPU.
"""
import numpy as np
import pytest

import oracle
from oracle import linear as Lm
from oracle import lloyd_max as LL
from oracle import quant as Qm
from oracle import rpbh as R

import test_oracle_linear as TL
import test_oracle_lloyd_max as TLL
import test_oracle_quant as TQ
import test_oracle_rpbh as TR


def _fails(fn, *a):
    try:
        return not fn(*a)
    except Exception:
        return True


def _rot_mutant(kind):
    def rotate(z, plan, h):
        z = np.asarray(z, dtype=np.float64)
        T, d = z.shape
        H = R.sylvester_hadamard(h).astype(np.float64)
        if kind != "no_norm":
            H = H / np.sqrt(h)
        for signs, perm in plan:
            if kind == "sign_by_source":
                u = (signs[None, :] * z)[:, perm]
            elif kind == "scatter":
                u = np.empty_like(z)
                u[:, perm] = signs[None, :] * z
            else:
                u = signs[None, :] * z[:, perm]
            if kind == "strided_blocks":
                z = (u.reshape(T, h, d // h).transpose(0, 2, 1) @ H.T)
                z = z.transpose(0, 2, 1).reshape(T, d)
            else:
                z = (u.reshape(T, d // h, h) @ H.T).reshape(T, d)
        return z
    return rotate


@pytest.mark.parametrize("kind", ["no_norm", "sign_by_source", "scatter", "strided_blocks"])
def test_rotation_mistakes_are_caught(monkeypatch, kind):
    monkeypatch.setattr(R, "rotate", _rot_mutant(kind))
    caught = (_fails(TR.check_orthogonal, 64, 16, 1)
              or _fails(TR.check_basis_closed_form, 32, 8)
              or _fails(TR.check_basis_closed_form, 64, 16))
    assert caught


def test_hadamard_sign_mistake_is_caught(monkeypatch):
    def bad(h):
        i = np.arange(h, dtype=np.uint64)
        par = np.bitwise_count(i[:, None] | i[None, :]) & 1
        return np.where(par == 1, -1, 1).astype(np.int64)
    monkeypatch.setattr(R, "sylvester_hadamard", bad)
    # (-1)^popcount(i|j) is D H D, still a Hadamard matrix: the Sylvester pins catch it
    assert _fails(TR.check_sylvester, 8)


def test_splitmix_mistake_is_caught(monkeypatch, golden_dir):
    def bad_mix(z):
        with np.errstate(over="ignore"):
            z = (z ^ (z >> np.uint64(29))) * R._M1
            z = (z ^ (z >> np.uint64(27))) * R._M2
            return z ^ (z >> np.uint64(31))
    monkeypatch.setattr(R, "_mix64", bad_mix)
    assert _fails(TR.check_splitmix_vector, golden_dir)


def test_absmax_mistakes_are_caught(monkeypatch):
    z = np.random.default_rng(1).standard_normal((20, 64))

    def off_by_one(z, qmax, eps=1e-10):
        r = np.max(np.abs(z), axis=1)
        alpha = np.maximum(r, eps) / (qmax + 1)
        return np.clip(np.rint(z / alpha[:, None]), -qmax, qmax).astype(np.int64), alpha

    def floor_round(z, qmax, eps=1e-10):
        r = np.max(np.abs(z), axis=1)
        alpha = np.maximum(r, eps) / qmax
        return np.clip(np.floor(z / alpha[:, None]), -qmax, qmax).astype(np.int64), alpha

    for m in (off_by_one, floor_round):
        monkeypatch.setattr(Qm, "absmax_quantize", m)
        assert _fails(TQ.check_absmax, z, 7)


def test_lloyd_max_code_mistake_is_caught(monkeypatch):
    z = np.random.default_rng(2).standard_normal((10, 64))

    def shifted(z, thresholds, eps=1e-10):
        sigma = np.maximum(np.sqrt(np.mean(z * z, axis=1)), eps)
        codes = np.searchsorted(thresholds, z / sigma[:, None], side="left")
        return np.minimum(codes + 1, 15), sigma

    monkeypatch.setattr(Qm, "lloyd_max_quantize", shifted)
    assert _fails(TQ.check_lloyd_max_codes, z)


def test_percentile_mistakes_are_caught(monkeypatch):
    z = np.random.default_rng(5).standard_normal((8, 3072)) * 2.0
    orig = Qm.percentile_quantize

    def no_normalisation(z, qmax, rho=Qm.PCT_RHO, gamma=Qm.PCT_GAMMA, eps=Qm.EPS):
        q = np.quantile(np.abs(z), rho, axis=1)
        alpha = np.maximum(gamma * q, eps) / qmax
        return np.clip(np.rint(z / alpha[:, None]), -qmax, qmax).astype(np.int64), alpha

    def order_statistic(z, qmax, rho=Qm.PCT_RHO, gamma=Qm.PCT_GAMMA, eps=Qm.EPS):
        q = np.quantile(np.abs(z), rho, axis=1, method="inverted_cdf")
        alpha = np.maximum(gamma * q / Qm.ndtri((1 + rho) / 2), eps) / qmax
        return np.clip(np.rint(z / alpha[:, None]), -qmax, qmax).astype(np.int64), alpha

    def no_clip(z, qmax, rho=Qm.PCT_RHO, gamma=Qm.PCT_GAMMA, eps=Qm.EPS):
        codes, alpha = orig(z, qmax, rho, gamma, eps)
        return np.rint(z / alpha[:, None]).astype(np.int64), alpha

    for m in (no_normalisation, order_statistic, no_clip):
        monkeypatch.setattr(Qm, "percentile_quantize", m)
        assert _fails(TQ.check_percentile, z)


def test_lloyd_iteration_mistake_is_caught(monkeypatch, golden_dir):
    def bad(levels=16, tol=1e-15, max_iter=2000):
        c = np.linspace(-2.5, 2.5, levels)
        for _ in range(max_iter):
            t = 0.5 * (c[:-1] + c[1:])
            e = np.concatenate(([-np.inf], t, [np.inf]))
            c = (LL._phi(e[:-1]) - LL._phi(e[1:]))          # forgot / P(cell)
        return c, 0.5 * (c[:-1] + c[1:])
    c, t = bad()
    assert _fails(TLL.check_conditions, c, t) and _fails(TLL.check_max1960, c, t, golden_dir)


def test_gemm_transpose_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(Lm, "gemm_int", lambda a, w: np.asarray(a, float) @ np.asarray(w, float))
    assert _fails(TL.check_gemm)


def test_dropped_rank1_term_is_caught(monkeypatch):
    def no_rank1(x, w, plan, h, center_tokens, bias=None):
        x = np.asarray(x, dtype=np.float64)
        xc = oracle.center(x)[0] if center_tokens else x
        y = Lm.rotate(xc, plan, h) @ Lm.rotate(np.asarray(w, float), plan, h).T
        return y + (0 if bias is None else np.asarray(bias)[None, :])
    monkeypatch.setattr(Lm, "linear_unquantized", no_rank1)
    assert _fails(TL.check_identity_quantizer, True, 1, False)


def test_weight_rotation_transposed_is_caught(monkeypatch):
    # weights rotated by Q instead of Q^T (rows through the inverse): W_R = W Q
    def bad(x, w, plan, h, center_tokens, bias=None):
        x = np.asarray(x, dtype=np.float64)
        w = np.asarray(w, dtype=np.float64)
        xc, mean = oracle.center(x) if center_tokens else (x, None)
        y = Lm.rotate(xc, plan, h) @ oracle.unrotate(w, plan, h).T
        if mean is not None:
            y = y + mean[:, None] * w.sum(axis=1)[None, :]
        return y + (0 if bias is None else np.asarray(bias)[None, :])
    monkeypatch.setattr(Lm, "linear_unquantized", bad)
    assert _fails(TL.check_identity_quantizer, False, 1, False)


# ---- grouped g = 64 weights ----------------------------------------------------------------

import test_oracle_weights_g64 as TG  # noqa: E402
from oracle import weights_g64 as Gm  # noqa: E402

_asym_ok = Gm.asym_group_quantize
_dequant_ok = Gm.dequantize
_corr_ok = Gm.corrected_product


def _asym_mutant(kind):
    def asym_group_quantize(w, g=Gm.GROUP, bits=4, store=None, eps=Gm.EPS):
        w = np.asarray(w, dtype=np.float64)
        n, d = w.shape
        top = 2 ** bits - 1
        wg = w.reshape(n, d // g, g)
        lo, hi = wg.min(axis=2), wg.max(axis=2)
        sigma = np.maximum(hi - lo, eps) / (top + 1 if kind == "step_over_16" else top)
        if store is not None:
            sigma = np.maximum(np.maximum(sigma, Gm.SIGMA_MIN_F16), np.abs(lo) / Gm.SHIFT_MAX)
            sigma = sigma.astype(store).astype(np.float64)
        z = (lo if kind == "shift_sign" else -lo) / sigma
        if store is not None:
            z = z.astype(store).astype(np.float64)
        rnd = np.floor if kind == "floor" else np.rint
        q = np.clip(rnd(wg / sigma[..., None] + z[..., None]), 0, top).astype(np.int64)
        return q.reshape(n, d), sigma, z
    return asym_group_quantize


def _pins_fail():
    for t in (TG.test_reconstruction_error_and_extremes, TG.test_codes_are_the_nearest_grid_point,
              TG.test_fp16_storage_codes_nearest_on_stored_grid,
              TG.test_layer_reduces_to_unquantized_for_fine_weights):
        if _fails(lambda: (t(), True)[1]):
            return True
    return False


@pytest.mark.parametrize("kind", ["shift_sign", "floor", "step_over_16"])
def test_grouped_quantizer_mistakes_are_caught(monkeypatch, kind):
    monkeypatch.setattr(Gm, "asym_group_quantize", _asym_mutant(kind))
    assert _pins_fail()


def test_grouped_dequantize_and_correction_mistakes_are_caught(monkeypatch):
    # sigma (Q + z) for sigma (Q - z)
    monkeypatch.setattr(Gm, "dequantize", lambda q, s, z, g=Gm.GROUP: _dequant_ok(q, s, -z, g))
    assert _pins_fail() or _fails(lambda: (TG.test_zero_point_correction_identity(), True)[1])
    monkeypatch.setattr(Gm, "dequantize", _dequant_ok)
    # z' = z instead of z - 8 in the App. B.2 correction
    monkeypatch.setattr(Gm, "corrected_product",
                        lambda a, q, s, z, g=Gm.GROUP: _corr_ok(a, q, s, z + 8.0, g))
    assert _fails(lambda: (TG.test_zero_point_correction_identity(), True)[1])


def test_a2_mistakes_are_caught(monkeypatch):
    # the 2-bit packing with the element order reversed inside a byte
    def bad_pack(v):
        v = np.asarray(v, dtype=np.int64) & 0x3
        return (v[..., 3::4] | (v[..., 2::4] << 2) | (v[..., 1::4] << 4)
                | (v[..., 0::4] << 6)).astype(np.uint8)
    with monkeypatch.context() as m:
        m.setattr(Qm, "pack_pairs", bad_pack)
        assert _fails(TQ.check_pairs)
    # the layer's A2 kind on the b-bit count 2^b - 1 = 3 instead of 2^(b-1) - 1 = 1
    real = Lm.percentile_quantize
    with monkeypatch.context() as m:
        m.setattr(Lm, "percentile_quantize", lambda z, qmax: real(z, 3 if qmax == 1 else qmax))
        assert _fails(TQ.check_layer_a2)
    # a ternary threshold at alpha instead of alpha / 2 (a floor instead of a rounding)
    def bad_pct(z, qmax, rho=Qm.PCT_RHO, gamma=Qm.PCT_GAMMA, eps=Qm.EPS):
        z = np.asarray(z, dtype=np.float64)
        q = np.quantile(np.abs(z), rho, axis=1)
        alpha = np.maximum(gamma * q / Qm.ndtri((1.0 + rho) / 2.0), eps) / qmax
        c = np.clip(np.trunc(z / alpha[:, None]), -qmax, qmax).astype(np.int64)
        return c, alpha
    with monkeypatch.context() as m:
        m.setattr(Qm, "percentile_quantize", bad_pct)
        assert _fails(TQ.check_ternary, np.random.default_rng(8).standard_normal((4, 1024)) * 2.0)
