"""The C-ABI library on the CPU: it loads, exports every declared entry point, and its
host-side tables agree with the oracle (no GPU needed, no compute call is made)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import w4a8_ptq_linear_b200 as oq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "oq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(oq_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from w4a8_ptq_linear_b200 import build
    build.build()
    return oq.lib()


def test_library_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    bound = {s[0] for s in oq.SIGNATURES}
    assert set(names) == bound, "binding and header disagree"


def test_checked_build_exports_the_same_symbols(lib):
    # the bounds-checked variant (-DOQ_CHECKED) is the same ABI
    from w4a8_ptq_linear_b200 import build
    path = build.build(checked=True)
    checked = oq.load(path)
    for n in declared_symbols():
        assert hasattr(checked, n), n


def test_status_strings(lib):
    for code, name in [(0, "OQ_OK"), (1, "OQ_ERR_INVALID_ARG"), (5, "OQ_ERR_DEVICE_TIMEOUT")]:
        assert lib.oq_status_string(code).decode() == name


@pytest.mark.parametrize("d,rounds,seed", [(256, 1, 0), (3072, 2, 0), (1920, 2, 7),
                                           (30720, 1, 123456789)])
def test_rpbh_tables_match_oracle_bit_for_bit(lib, d, rounds, seed):
    plan = oracle.rpbh_plan(d, oracle.default_block(d) if d % 1024 == 0 else 64, rounds, seed)
    for r in range(rounds):
        s, p = oq.rpbh_tables(d, r, seed)
        assert np.array_equal(s.astype(np.float64), plan[r][0])
        assert np.array_equal(p.astype(np.int64), plan[r][1])


def test_newton_codebook_matches_lloyd_iteration(lib):
    c_lib, t_lib = oq.lloyd_max_codebook()
    c_or, t_or = oracle.lloyd_max_gaussian()
    assert np.abs(c_lib - c_or).max() < 1e-10
    assert np.abs(t_lib - t_or).max() < 1e-10


def test_width_codebook_matches_lloyd_iteration(lib):
    # library: Newton with Simpson cell probabilities; oracle: Lloyd iteration with the
    # incomplete beta function
    for d in (32, 256, 1920, 3072, 30720):
        c, t = oq.lloyd_max_codebook_width(d)
        c_or, t_or = oracle.lloyd_max_sphere(d)
        assert np.abs(c - c_or).max() < 1e-8 and np.abs(t - t_or).max() < 1e-8, d
    assert lib.oq_lloyd_max_codebook_width(16, None, None) == oq.OQ_ERR_INVALID_ARG


def test_codebook_256_matches_lloyd_iteration(lib):
    c, t = oq.lloyd_max_codebook_8bit()
    c_or, t_or = oracle.lloyd_max_gaussian_8bit()
    assert np.abs(c - c_or).max() < 1e-8 and np.abs(t - t_or).max() < 1e-8
    h = ctypes.c_void_p()
    assert lib.oq_plan_create(ctypes.byref(h), 16384, 1024, 1, 0, 0, 5) == oq.OQ_ERR_UNSUPPORTED


def test_default_policies_match_oracle(lib):
    for d in (256, 1152, 1920, 3072, 4096, 30720):
        assert oq.default_block(d) == oracle.default_block(d)
    for h in (64, 128, 256, 512, 1024):
        assert oq.default_rounds(h) == oracle.default_rounds(h)


def test_argument_validation_before_any_cuda_call(lib):
    h = ctypes.c_void_p()
    # h does not divide d, h not a power of two, bad rounds, bad d: rejected up front
    for args in [(3072, 2048, 1), (3072, 96, 1), (3072, 1024, 3), (3000, 8, 1), (0, 8, 1)]:
        st = lib.oq_plan_create(ctypes.byref(h), args[0], args[1], args[2], 0, 0, 0)
        assert st == oq.OQ_ERR_INVALID_ARG, args
    st = lib.oq_plan_create(ctypes.byref(h), 256, 64, 1, 0, 0, 9)
    assert st == oq.OQ_ERR_INVALID_ARG
    # the percentile scale keeps at most 6 order statistics per token: d <= 8192
    st = lib.oq_plan_create(ctypes.byref(h), 16384, 1024, 1, 0, 0, 3)
    assert st == oq.OQ_ERR_UNSUPPORTED
    assert b"percentile" in lib.oq_last_error()
    # GEMM shape checks happen before any launch
    st = lib.oq_gemm_w4a8(None, None, None, None, None, None, None, 16, 100, 256, 0, None, None)
    assert st == oq.OQ_ERR_INVALID_ARG
    assert b"d_in" in lib.oq_last_error()


def test_grouped_weight_arguments_rejected_up_front(lib):
    # grouped (g = 64) weights: activation kind, d_in % 64 and w_sz are checked before any launch
    st = lib.oq_gemm_w4a4_g64(oq.ACT_KINDS["int4_lloydmax"], None, None, None, None, None, None,
                              None, None, 16, 256, 256, 0, None, None)
    assert st == oq.OQ_ERR_INVALID_ARG
    assert b"INT4_ABSMAX" in lib.oq_last_error()
    st = lib.oq_gemm_w4a4_g64(oq.ACT_KINDS["int4_absmax"], None, None, None, None, None, None,
                              None, None, 16, 96, 256, 0, None, None)
    assert st == oq.OQ_ERR_INVALID_ARG
    assert b"64" in lib.oq_last_error()
    st = lib.oq_gemm_w4a4_g64(oq.ACT_KINDS["int4_absmax"], None, None, None, None, None, None,
                              None, None, 16, 256, 256, 0, None, None)
    assert st == oq.OQ_ERR_INVALID_ARG
    assert b"w_sz" in lib.oq_last_error()
    assert lib.oq_prepare_weights_g64(None, None, 16, 256, None, None, None, None,
                                      None) == oq.OQ_ERR_INVALID_ARG
    assert lib.oq_linear_g64(None, None, 16, 256, None, None, None, None, None, 256, None, None,
                             0, None) == oq.OQ_ERR_INVALID_ARG


def _gather_position(h, t, i):
    """Rotated position that thread t, register i of a round's gather holds (the block
    transform's arrangement: consecutive for h <= 128, strided within the warp's 1024 positions
    for h >= 256)."""
    if h <= 128:
        return t * 32 + i
    e2 = h // 32
    w, lane = divmod(t, 32)
    blk, kb = divmod(lane, e2)
    ia, ib = divmod(i, e2)
    return w * 1024 + blk * h + kb + e2 * ia + 32 * ib


@pytest.mark.parametrize("d,h,seed", [(256, 64, 0), (3072, 1024, 0), (1920, 128, 0),
                                      (1920, 64, 3), (4096, 256, 11), (8192, 512, 5),
                                      (1280, 256, 0), (96, 32, 2), (32, 1, 9)])
def test_pair_word_layout_is_bank_conflict_free(lib, d, h, seed):
    # every warp-wide store of the interleave pass and every warp-wide round-1 gather touches
    # distinct banks (bank = word % 32), and the words of distinct channels are distinct
    word = oq.debug_pair_layout(d, h, seed)
    nact = d // 32
    nwarps = (nact + 31) // 32
    assert len(set(word.tolist())) == d and word.min() >= 0 and word.max() < nwarps * 1024
    bank = word % 32
    for w in range(nwarps):
        lanes = [t for t in range(32 * w, min(32 * w + 32, nact))]
        for m in range(4):
            for k in range(8):
                chans = [8 * (t + m * nact) + k for t in lanes]
                assert len(set(bank[chans].tolist())) == len(chans)
    perm = oracle.rpbh_plan(d, h, 1, seed)[0][1].astype(np.int64)
    for w in range(nwarps):
        lanes = [t for t in range(32 * w, min(32 * w + 32, nact))]
        for i in range(32):
            chans = [perm[_gather_position(h, t, i)] for t in lanes]
            assert len(set(bank[chans].tolist())) == len(chans)
