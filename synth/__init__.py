"""Seeded synthetic inputs for the rotated, quantized linear layer.

This module only draws numbers. It holds none of the method's arithmetic: no rotation,
no quantizer, no GEMM. Both the CPU oracle (through the tests and the bench) and the CUDA
library are fed from it, and neither of them imports the other.

Every tensor is drawn in float64 with ``numpy.random.default_rng(seed)`` and rounded to
bfloat16 (round-to-nearest-even), which is the storage type of activations and weights.
Values are returned as ``uint16`` bfloat16 bit patterns; ``bf16_to_f64`` decodes them
exactly.

Workloads (the distributions of the layers the pages study: DiT widths 3072 and 1920 with an
adaptive-layer-norm per-token mean, widths up to 30720; CentriQ §4.1 "DC energy in DiT
activations", OrbitQuant PR #25 "Benchmark subsets"):

- ``tiny``      T=64, d=256, N=256, h=64, 1 round, A8; X ~ N(0,1) + per-token mean
                N(0, var 2), four outlier channels scaled x20; W ~ N(0, 1/d).
- ``dit_w4a8``  T=4096, d=N=3072, h=1024, 1 round, A8; X ~ N(0,1) with 1% of entries replaced
                by Student-t(3) draws, plus a per-token mean N(0, var 3); W ~ N(0, 1/d).
- ``dit_a4``    the ``dit_w4a8`` layer with centered A4 absmax activations (CentriQ's W4A4).
- ``narrow_lm`` T=8192, d=N=1920, h=128, 2 rounds, A4 Lloyd-Max; X and W as ``dit_w4a8``.
- ``mlp_up``    T=4096, d=3072, N=12288, h=1024, 1 round, centered A4 absmax; X ~ N(0,1)
                + per-token mean N(0, var 5); W ~ N(0, 1/d).
- ``sweep``     rotate+quantize only; X as ``dit_w4a8`` at any (T, d).

The second parameter of every N(., .) above is a variance.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "f64_to_bf16", "bf16_to_f64", "make_x", "make_x_parallel", "make_w",
    "make_bias", "make_inputs", "sweep_points",
]


def f64_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 bit patterns (round to nearest, ties to even).

    The value is first rounded to float32 by numpy (RNE), then the low 16 bits are rounded
    away with ties to even. Non-finite values are not produced by the generators (for finite
    values the 32-bit sum below cannot wrap).
    """
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    """Decode bfloat16 bit patterns exactly to float64."""
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    n_out: int
    h: int
    rounds: int
    act: str            # "int8_absmax" | "int4_absmax" | "int4_lloydmax" | "int4_percentile"
                        # | "int4_lloydmax_width" | "int8_lloydmax" | "int2_percentile"
    center: bool
    mean_var: float     # variance of the per-token mean offset
    outliers: int = 0   # channels scaled by outlier_gain (tiny workload)
    outlier_gain: float = 20.0
    heavy_frac: float = 0.0   # fraction of N(0,1) entries replaced by Student-t(3)
    seed: int = 0
    weights: str = "int4_channel"   # "int4_channel" (symmetric per output channel) | "int4_g64"
    notes: str = field(default="", compare=False)


WORKLOADS = {
    "tiny": Workload("tiny", 64, 256, 256, 64, 1, "int8_absmax", False, 2.0, outliers=4),
    "dit_w4a8": Workload("dit_w4a8", 4096, 3072, 3072, 1024, 1, "int8_absmax", False, 3.0,
                         heavy_frac=0.01),
    # the DiT-width layer with 8-bit Lloyd-Max activations (the A8 alternative that OrbitQuant
    # PR #25 compares absmax INT8 against)
    "dit_lm8": Workload("dit_lm8", 4096, 3072, 3072, 1024, 1, "int8_lloydmax", False, 3.0,
                        heavy_frac=0.01),
    # the same layer with CentriQ's centered INT4 activations (W4A4)
    "dit_a4": Workload("dit_a4", 4096, 3072, 3072, 1024, 1, "int4_absmax", True, 3.0,
                       heavy_frac=0.01),
    "narrow_lm": Workload("narrow_lm", 8192, 1920, 1920, 128, 2, "int4_lloydmax", False, 3.0,
                          heavy_frac=0.01),
    # the same layer with the width-d codebook (per-width tables, codebook v3)
    "narrow_lm_w": Workload("narrow_lm_w", 8192, 1920, 1920, 128, 2, "int4_lloydmax_width", False,
                            3.0, heavy_frac=0.01),
    "mlp_up": Workload("mlp_up", 4096, 3072, 12288, 1024, 1, "int4_absmax", True, 5.0),
    # the same layer with CentriQ's percentile per-token scale (§4.2 "Scale and grid")
    "mlp_up_pct": Workload("mlp_up_pct", 4096, 3072, 12288, 1024, 1, "int4_percentile", True,
                           5.0),
    # the same layer with 2-bit activations (CentriQ's W4A2: grid {-1, 0, 1}, percentile scale)
    "mlp_up_a2": Workload("mlp_up_a2", 4096, 3072, 12288, 1024, 1, "int2_percentile", True, 5.0),
    # the same layer with CentriQ's weight format: asymmetric INT4 groups of 64 columns (§4.3)
    "mlp_up_g64": Workload("mlp_up_g64", 4096, 3072, 12288, 1024, 1, "int4_absmax", True, 5.0,
                           weights="int4_g64"),
}


def _rng(seed: int, stream: int) -> np.random.Generator:
    # independent streams for X, W and bias so that changing T does not change W
    return np.random.default_rng([seed, stream])


def make_x(T: int, d: int, *, mean_var: float, heavy_frac: float = 0.0, outliers: int = 0,
           outlier_gain: float = 20.0, seed: int = 0, row_offset: int = 0) -> np.ndarray:
    """Activations [T, d] as bfloat16 bits.

    Rows are drawn independently per token from a generator keyed on (seed, row block), so
    a row range can be regenerated without drawing the rows before it (``row_offset``).
    """
    out = np.empty((T, d), dtype=np.uint16)
    chan_rng = _rng(seed, 7)
    outlier_ch = chan_rng.permutation(d)[:outliers] if outliers else None
    BLK = 256
    t = 0
    while t < T:
        g0 = (row_offset + t) // BLK
        lo = (row_offset + t) - g0 * BLK
        n = min(BLK - lo, T - t)
        rng = np.random.default_rng([seed, 1, g0])
        base = rng.standard_normal((BLK, d))
        if heavy_frac > 0.0:
            mask = rng.random((BLK, d)) < heavy_frac
            base[mask] = rng.standard_t(3.0, size=int(mask.sum()))
        mu = rng.standard_normal((BLK, 1)) * np.sqrt(mean_var)
        x = base + mu
        if outlier_ch is not None:
            x[:, outlier_ch] *= outlier_gain
        out[t:t + n] = f64_to_bf16(x[lo:lo + n])
        t += n
    return out


def _fill_rows(job):
    # worker of make_x_parallel: rows [r0, r1) of the shared array
    from multiprocessing import shared_memory
    name, T, d, r0, r1, kw = job
    shm = shared_memory.SharedMemory(name=name)
    try:
        arr = np.ndarray((T, d), dtype=np.uint16, buffer=shm.buf)
        arr[r0:r1] = make_x(r1 - r0, d, row_offset=r0, **kw)
        del arr
    finally:
        shm.close()
    return r1 - r0


def make_x_parallel(T: int, d: int, *, workers: int | None = None, **kw) -> np.ndarray:
    """``make_x(T, d, **kw)`` drawn by a pool of processes (the same bits: rows come from
    generators keyed on their row block). The pool uses the spawn start method, which is safe
    after CUDA has been initialised in the calling process."""
    import multiprocessing as mp
    import os
    from multiprocessing import shared_memory
    workers = workers or min(32, os.cpu_count() or 1)
    if workers <= 1 or T * d < (1 << 24):
        return make_x(T, d, **kw)
    blk = 256 * max(1, -(-T // (256 * 4 * workers)))     # whole row blocks, ~4 jobs per worker
    shm = shared_memory.SharedMemory(create=True, size=max(1, T * d * 2))
    try:
        jobs = [(shm.name, T, d, r, min(T, r + blk), kw) for r in range(0, T, blk)]
        with mp.get_context("spawn").Pool(workers) as pool:
            assert sum(pool.map(_fill_rows, jobs)) == T
        return np.ndarray((T, d), dtype=np.uint16, buffer=shm.buf).copy()
    finally:
        shm.close()
        shm.unlink()


def make_w(n_out: int, d: int, *, seed: int = 0) -> np.ndarray:
    """Weights [n_out, d] ~ N(0, 1/d) as bfloat16 bits."""
    rng = _rng(seed, 2)
    return f64_to_bf16(rng.standard_normal((n_out, d)) / np.sqrt(d))


def make_bias(n_out: int, *, seed: int = 0, scale: float = 0.1) -> np.ndarray:
    """Bias [n_out] ~ N(0, scale^2) as bfloat16 bits (the workloads use no bias by default)."""
    rng = _rng(seed, 3)
    return f64_to_bf16(rng.standard_normal(n_out) * scale)


def make_inputs(name: str, *, T: int | None = None, seed: int | None = None):
    """(workload, X bits [T, d], W bits [N, d]) for a named workload, T optionally cut."""
    wl = WORKLOADS[name]
    T = wl.T if T is None else T
    seed = wl.seed if seed is None else seed
    x = make_x(T, wl.d, mean_var=wl.mean_var, heavy_frac=wl.heavy_frac,
               outliers=wl.outliers, outlier_gain=wl.outlier_gain, seed=seed)
    w = make_w(wl.n_out, wl.d, seed=seed)
    return wl, x, w


def sweep_points():
    """The rotate+quantize bandwidth sweep: (T, d, h, rounds, act) tuples, h | d."""
    pts = []
    for T in (256, 4096, 65536):
        for d in (1920, 3072, 4096, 30720):
            for h in (64, 128, 256, 512, 1024):
                if d % h:
                    continue
                for rounds in (1, 2):
                    for act in ("int8_absmax", "int4_lloydmax"):
                        pts.append((T, d, h, rounds, act))
    return pts
