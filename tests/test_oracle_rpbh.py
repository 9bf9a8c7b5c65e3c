"""Pins for the oracle's RPBH rotation (CPU only).

Each check ties the oracle to something other than itself: the algebra of Hadamard matrices
(CentriQ §3 "Hadamard rotation", Lemma 1, App. C.5), a closed form for rotated basis vectors,
and a published SplitMix64 output sequence. The ``check_*`` helpers are reused by
test_oracle_mutations.py to show that planted mistakes are caught.
"""
import os

import numpy as np
import pytest

import oracle
from oracle import rpbh as R


def check_splitmix_vector(golden_dir):
    want = [int(l) for l in open(os.path.join(golden_dir, "splitmix64_seed1234567.txt"))
            if l.strip() and not l.startswith("#")]
    got = [int(v) for v in R.splitmix64_at(np.uint64(1234567), np.arange(len(want)))]
    return got == want


def check_hadamard(h):
    H = R.sylvester_hadamard(h)
    return bool(np.array_equal(H @ H.T, h * np.eye(h, dtype=np.int64))
                and np.array_equal(H, H.T))


def check_sylvester(h):
    """Hadamard, and the Sylvester one: equal to the Kronecker recursion, row sums h e_1."""
    H = R.sylvester_hadamard(h)
    s = H.sum(axis=1)
    return (check_hadamard(h) and bool(np.array_equal(H, kron_hadamard(h)))
            and s[0] == h and bool(np.all(s[1:] == 0)))


def kron_hadamard(h):
    """Sylvester's recursion H_{2n} = [[H_n, H_n], [H_n, -H_n]], independent of popcount."""
    H = np.ones((1, 1), dtype=np.int64)
    while H.shape[0] < h:
        H = np.block([[H, H], [H, -H]])
    return H


def check_orthogonal(d, h, rounds, seed=0):
    plan = R.rpbh_plan(d, h, rounds, seed)
    Q = R.rpbh_matrix(d, plan, h)
    return float(np.abs(Q.T @ Q - np.eye(d)).max()) < 1e-12


def check_basis_closed_form(d, h, seed=3):
    """One round maps e_j to (s[i] / sqrt(h)) * column (i mod h) of H_h in block i // h,
    where i is the gathered position that reads channel j (pi[i] = j)."""
    plan = R.rpbh_plan(d, h, 1, seed)
    signs, perm = plan[0]
    H = kron_hadamard(h).astype(np.float64)
    inv = np.empty(d, dtype=np.int64)
    inv[perm] = np.arange(d)
    got = R.rotate(np.eye(d), plan, h)
    want = np.zeros((d, d))
    for j in range(d):
        i = inv[j]
        b, m = divmod(i, h)
        want[j, b * h:(b + 1) * h] = signs[i] * H[:, m] / np.sqrt(h)
    return float(np.abs(got - want).max()) < 1e-14


def test_splitmix64_published_sequence(golden_dir):
    assert check_splitmix_vector(golden_dir)


@pytest.mark.parametrize("h", [1, 2, 4, 8, 16, 64, 128, 256, 1024])
def test_hadamard_is_hadamard(h):
    assert check_hadamard(h)


@pytest.mark.parametrize("h", [2, 8, 64, 1024])
def test_popcount_form_equals_kronecker_recursion(h):
    assert check_sylvester(h)


@pytest.mark.parametrize("h", [2, 4, 64, 1024])
def test_sylvester_row_sums_lemma1(h):
    # CentriQ Lemma 1 / App. C.5: one row of H_{2^k} sums to 2^k, every other to 0,
    # so H 1 = 2^k e_1 and no Sylvester matrix of order >= 2 is regular.
    s = R.sylvester_hadamard(h).sum(axis=1)
    assert s[0] == h and np.all(s[1:] == 0)


@pytest.mark.parametrize("d,h,rounds", [(64, 8, 1), (256, 64, 1), (256, 64, 2), (192, 64, 2),
                                        (128, 128, 1), (96, 1, 1)])
def test_rpbh_is_orthogonal(d, h, rounds):
    assert check_orthogonal(d, h, rounds)


@pytest.mark.parametrize("d,h", [(32, 8), (64, 16), (48, 16)])
def test_rotated_basis_closed_form(d, h):
    assert check_basis_closed_form(d, h)


def test_rotate_preserves_norm_and_inverts():
    rng = np.random.default_rng(11)
    for d, h, rounds in [(256, 64, 1), (1920, 128, 2), (3072, 1024, 1)]:
        x = rng.standard_normal((5, d)) * rng.uniform(0.1, 10, (5, 1))
        plan = R.rpbh_plan(d, h, rounds, 0)
        z = R.rotate(x, plan, h)
        assert np.allclose(np.linalg.norm(z, axis=1), np.linalg.norm(x, axis=1),
                           rtol=1e-13, atol=0)
        assert np.abs(R.unrotate(z, plan, h) - x).max() < 1e-12 * np.abs(x).max()


def test_plan_is_deterministic_valid_and_rounds_independent():
    d = 3072
    p1 = R.rpbh_plan(d, 1024, 2, 0)
    p2 = R.rpbh_plan(d, 1024, 2, 0)
    for (s1, q1), (s2, q2) in zip(p1, p2):
        assert np.array_equal(s1, s2) and np.array_equal(q1, q2)
        assert set(np.unique(s1)) <= {-1.0, 1.0}
        assert np.array_equal(np.sort(q1), np.arange(d))
    assert not np.array_equal(p1[0][1], p1[1][1])
    assert not np.array_equal(p1[0][0], p1[1][0])
    p3 = R.rpbh_plan(d, 1024, 1, 1)
    assert not np.array_equal(p1[0][1], p3[0][1])
    # the first round does not depend on how many rounds are drawn
    p4 = R.rpbh_plan(d, 1024, 1, 0)
    assert np.array_equal(p4[0][1], p1[0][1]) and np.array_equal(p4[0][0], p1[0][0])


def test_signs_balanced_and_permutation_uniform():
    # signs: a fair coin; |#(-1) - d/2| well inside 5 standard deviations
    s, _ = R.rpbh_plan(30720, 1024, 1, 0)[0]
    neg = int((s < 0).sum())
    assert abs(neg - 15360) < 5 * np.sqrt(30720 / 4)
    # permutation: where channel 0 lands, over many seeds, is uniform (chi-square)
    d, n = 16, 4000
    counts = np.zeros(d)
    for seed in range(n):
        perm = R.rpbh_plan(d, 16, 1, seed)[0][1]
        counts[int(np.nonzero(perm == 0)[0][0])] += 1
    chi2 = float(((counts - n / d) ** 2 / (n / d)).sum())
    assert chi2 < 45.0      # 15 dof: P(chi2 > 45) is about 7e-5


def test_default_policies():
    # model card: largest power of two dividing the width; PR #25: 2 rounds when h < 512
    assert R.default_block(3072) == 1024
    assert R.default_block(1920) == 128
    assert R.default_block(4096) == 1024      # capped at the 1024 design limit
    assert R.default_block(1152) == 128
    assert R.default_rounds(128) == 2 and R.default_rounds(512) == 1
