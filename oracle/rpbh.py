"""Random-sign, permuted block Hadamard (RPBH) rotation -- oracle (test infrastructure).

What the pages fix:
- OrbitQuant PR #25, "Default changes": activations are pre-rotated by RPBH with block h; the
  "auto" policy adds an independent second RPBH round where h < 512.
- FLUX.1-schnell-OrbitQuant-W4A4 model card, "Quantization": rotation ``rpbh``, rotation
  seed 0, block size = the largest power of two dividing the width.
- CentriQ §3 "Hadamard rotation": H_n H_n^T = n I, so H_n / sqrt(n) is orthogonal and can be
  folded into the weight, W x = (W H^T)(H x); Sylvester matrices exist at every order 2^k.
  CentriQ §2 describes OrbitQuant's basis as block-Hadamard under a random permutation.

What the pages leave open, and the reading taken here (the library follows the same spec):
- One round is  z <- (I_{d/h} (x) H_h / sqrt(h)) . D_r . P_r . z,  with the permutation applied
  first as a gather, u_i = s_r[i] * z[pi_r[i]], then the signs (indexed by the gathered
  position), then the orthonormal Sylvester block transform on consecutive blocks of h.
- Signs and permutations come from SplitMix64 (Steele, Lea and Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014), used in counter form: output number i
  (0-based) of a generator seeded with ``key`` is  mix64(key + (i + 1) * 0x9E3779B97F4A7C15)
  with the published finaliser mix64. Round r (0-based) draws its sign stream from key
  value(seed, 2r) and its permutation stream from key value(seed, 2r + 1).
  s_r[i] = -1 when bit 63 of value(k_sign, i) is set, else +1.
  pi_r = the indices 0..d-1 sorted by value(k_perm, i), ties by the smaller index.
- The Sylvester matrix is H_h[i, j] = (-1)^popcount(i & j) (natural order).

Parity: pinned (tests/test_oracle_rpbh.py): H H^T = h I and the Kronecker recursion; the
row-sum property of Lemma 1; Q^T Q = I; inverse(rotate(x)) = x; a closed form for rotated
basis vectors that fixes the order of gather, sign and block transform; a published SplitMix64
output sequence.
"""
from __future__ import annotations

import numpy as np

GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output finaliser (Steele, Lea and Flood 2014)."""
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def splitmix64_at(key, idx) -> np.ndarray:
    """Output number ``idx`` (0-based) of a SplitMix64 generator seeded with ``key``."""
    key = np.asarray(key, dtype=np.uint64)
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = key + (idx + np.uint64(1)) * GOLDEN_GAMMA
    return _mix64(z)


def default_block(d: int) -> int:
    """Largest power of two dividing d (model card: block size policy), capped at 1024
    (the exported dense blocks go up to 1024, OrbitQuant PR #25 "Runtime work")."""
    h = d & -d
    return min(h, 1024)


def default_rounds(h: int) -> int:
    """OrbitQuant PR #25, "Default changes": a second independent round when h < 512."""
    return 2 if h < 512 else 1


def rpbh_plan(d: int, h: int, rounds: int, seed: int = 0):
    """Signs and permutations of every round: list of (signs float64[d], perm int64[d])."""
    if h <= 0 or h & (h - 1) or d % h:
        raise ValueError("h must be a power of two dividing d")
    idx = np.arange(d, dtype=np.uint64)
    plan = []
    for r in range(rounds):
        k_sign = splitmix64_at(np.uint64(seed), np.uint64(2 * r))
        k_perm = splitmix64_at(np.uint64(seed), np.uint64(2 * r + 1))
        vs = splitmix64_at(k_sign, idx)
        signs = np.where((vs >> np.uint64(63)) != 0, -1.0, 1.0)
        vp = splitmix64_at(k_perm, idx)
        perm = np.argsort(vp, kind="stable").astype(np.int64)   # ties keep index order
        plan.append((signs, perm))
    return plan


def sylvester_hadamard(h: int) -> np.ndarray:
    """Dense Sylvester Hadamard matrix, H[i, j] = (-1)^popcount(i & j), as int64."""
    i = np.arange(h, dtype=np.uint64)
    par = np.bitwise_count(i[:, None] & i[None, :]) & 1
    return np.where(par == 1, -1, 1).astype(np.int64)


def rotate(z: np.ndarray, plan, h: int) -> np.ndarray:
    """Apply every RPBH round to the rows of z (float64 [T, d]); returns float64 [T, d]."""
    z = np.asarray(z, dtype=np.float64)
    T, d = z.shape
    H = sylvester_hadamard(h).astype(np.float64) / np.sqrt(h)
    for signs, perm in plan:
        u = signs[None, :] * z[:, perm]                   # gather, then sign
        z = (u.reshape(T, d // h, h) @ H.T).reshape(T, d)  # block-diagonal H_h / sqrt(h)
    return z


def unrotate(y: np.ndarray, plan, h: int) -> np.ndarray:
    """Inverse of ``rotate``: every round undone in reverse order (Q^T y)."""
    y = np.asarray(y, dtype=np.float64)
    T, d = y.shape
    H = sylvester_hadamard(h).astype(np.float64) / np.sqrt(h)
    for signs, perm in reversed(plan):
        v = (y.reshape(T, d // h, h) @ H).reshape(T, d)   # H^T = H^{-1} for orthonormal H
        v = v * signs[None, :]
        y = np.empty_like(v)
        y[:, perm] = v                                     # scatter undoes the gather
    return y


def rpbh_matrix(d: int, plan, h: int) -> np.ndarray:
    """The dense d x d operator Q with rotate(x) = x @ Q^T (rows of Q = rotated basis)."""
    return rotate(np.eye(d), plan, h).T
