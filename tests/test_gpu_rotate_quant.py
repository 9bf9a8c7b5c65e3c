"""GPU parity of the fused center + RPBH + quantize kernel against the oracle.

Each case runs oq_rotate_quantize through the C ABI on seeded synthetic tokens and compares
element by element with the oracle: normalised rotated values (<= 1e-5 relative per token),
per-token scales (<= 1e-5 relative), means, and codes (identical except within 1e-5
relative of a decision boundary). Shapes span several CTAs' worth of tokens, ragged token
counts, every block size from 1 to 1024, one and two rounds and the widest width.
"""
import numpy as np
import pytest

import oracle
import synth
from parity import (ROT_TOL, absmax_boundary_mask, compare_codes, lloyd_max_boundary_mask,
                    per_token_rel, to_torch_bf16)

pytestmark = pytest.mark.gpu

QMAX = {"int8_absmax": 127, "int4_absmax": 7}

CASES = [
    # T, d, h, rounds, act, center
    (64, 256, 64, 1, "int8_absmax", False),
    (300, 3072, 1024, 1, "int8_absmax", False),
    (257, 3072, 1024, 1, "int4_absmax", True),
    (130, 1920, 128, 2, "int4_lloydmax", False),
    (77, 4096, 512, 1, "int8_absmax", True),
    (45, 4096, 256, 2, "int4_absmax", False),
    (33, 256, 1, 1, "int8_absmax", False),
    (40, 512, 8, 2, "int4_lloydmax", True),
    (1, 3072, 1024, 1, "int8_absmax", True),
    (9, 30720, 1024, 1, "int8_absmax", False),
    (5, 30720, 64, 2, "int4_lloydmax", True),
    (600, 1920, 64, 2, "int8_absmax", False),
    (4, 30720, 32, 1, "int4_absmax", True),
    (3, 30720, 512, 2, "int8_absmax", False),
    (70, 2048, 256, 1, "int4_lloydmax", True),
    (20, 1280, 256, 2, "int8_absmax", True),
    # CentriQ percentile scale: the quantile needs the R = d - floor(0.9995 (d - 1)) largest
    # magnitudes, R = 2 (d < 2000), 3, 4, 5, 6 (d = 8192)
    (257, 3072, 1024, 1, "int4_percentile", True),
    (130, 1920, 128, 2, "int4_percentile", False),
    (45, 4096, 256, 2, "int4_percentile", False),
    (31, 6144, 1024, 1, "int4_percentile", True),
    (20, 8192, 512, 1, "int4_percentile", True),
    (7, 256, 64, 1, "int4_percentile", False),
    # 2-bit activations (CentriQ W4A2: the percentile range, grid {-1, 0, 1}, four codes a byte)
    (257, 3072, 1024, 1, "int2_percentile", True),
    (130, 1920, 128, 2, "int2_percentile", False),
    (45, 4096, 256, 2, "int2_percentile", True),
    (20, 8192, 512, 1, "int2_percentile", True),
    (7, 256, 64, 1, "int2_percentile", False),
    (301, 1024, 1, 1, "int2_percentile", False),
    # the width-d Lloyd-Max codebook (codebook v3 tables per width)
    (130, 1920, 128, 2, "int4_lloydmax_width", False),
    (33, 256, 32, 1, "int4_lloydmax_width", True),
    (5, 30720, 1024, 1, "int4_lloydmax_width", False),
    # 8-bit Lloyd-Max codes (255 thresholds, binary search)
    (300, 3072, 1024, 1, "int8_lloydmax", False),
    (45, 4096, 256, 2, "int8_lloydmax", True),
    (7, 256, 64, 1, "int8_lloydmax", False),
]


def run_case(T, d, h, rounds, act, center, seed=0):
    import torch
    import w4a8_ptq_linear_b200 as oq
    xb = synth.make_x(T, d, mean_var=3.0, heavy_frac=0.01, seed=seed)
    plan = oq.Plan(d, h, rounds, seed=seed, center=center, act=act)
    x = to_torch_bf16(xb)
    codes, scale, mean, rot = oq.rotate_quantize(plan, x, rotated=True)
    torch.cuda.synchronize()
    st, code = oq.device_status()
    assert st == 0, code
    thresholds = (oracle.lloyd_max_sphere(d)[1] if act == "int4_lloydmax_width"
                  else oracle.lloyd_max_gaussian_8bit()[1] if act == "int8_lloydmax"
                  else oracle.lloyd_max_gaussian()[1])
    ref = oracle.quantize_activations(synth.bf16_to_f64(xb), oracle.rpbh_plan(d, h, rounds, seed),
                                      h, act, center, thresholds)
    out = {
        "codes": codes.cpu().numpy(), "scale": scale.cpu().numpy().astype(np.float64),
        "mean": None if mean is None else mean.cpu().numpy().astype(np.float64),
        "rot": rot.cpu().numpy().astype(np.float64),
    }
    plan.close()
    return xb, ref, out


@pytest.mark.parametrize("T,d,h,rounds,act,center", CASES)
def test_rotate_quantize_matches_oracle(T, d, h, rounds, act, center):
    xb, ref, out = run_case(T, d, h, rounds, act, center)
    # rotated values
    assert per_token_rel(out["rot"], ref["rotated"]).max() <= ROT_TOL
    # scales and means
    assert np.abs(out["scale"] / ref["scale"] - 1).max() <= ROT_TOL
    if center:
        x = synth.bf16_to_f64(xb)
        tol = 1e-6 * np.abs(x).mean(axis=1) + 1e-30
        assert np.all(np.abs(out["mean"] - ref["mean"]) <= tol)
    # codes
    if act == "int8_absmax":
        gpu = out["codes"].view(np.int8).astype(np.int64)
        ex = absmax_boundary_mask(ref["rotated"], ref["scale"], 127)
    elif act == "int8_lloydmax":
        gpu = out["codes"].view(np.uint8).astype(np.int64)
        ex = lloyd_max_boundary_mask(ref["rotated"], ref["scale"],
                                     oracle.lloyd_max_gaussian_8bit()[1])
    elif act in ("int4_absmax", "int4_percentile"):
        gpu = oracle.unpack_nibbles(out["codes"], signed=True)
        ex = absmax_boundary_mask(ref["rotated"], ref["scale"], 7)
    elif act == "int2_percentile":
        assert out["codes"].shape == (T, d // 4)
        gpu = oracle.unpack_pairs(out["codes"])
        ex = absmax_boundary_mask(ref["rotated"], ref["scale"], 1)
    else:
        gpu = oracle.unpack_nibbles(out["codes"], signed=False)
        thr = (oracle.lloyd_max_sphere(d)[1] if act == "int4_lloydmax_width"
               else oracle.lloyd_max_gaussian()[1])
        ex = lloyd_max_boundary_mask(ref["rotated"], ref["scale"], thr)
    bad, n_ex = compare_codes(gpu, ref["codes"], ex)
    assert bad == 0, f"{bad} codes differ outside the boundary exemption ({n_ex} exempt)"


# Every (width, block, rounds, output) point of the rotate+quantize bandwidth sweep, at a
# small odd token count (the two-token kernel's tail pass included): the sweep's token counts
# only change how many passes each CTA makes.
SWEEP = sorted({(d, h, rounds, act) for (_, d, h, rounds, act) in synth.sweep_points()})


@pytest.mark.parametrize("d,h,rounds,act", SWEEP)
def test_sweep_grid_matches_oracle(d, h, rounds, act):
    test_rotate_quantize_matches_oracle(9, d, h, rounds, act, False)


def test_zero_and_constant_tokens():
    import torch
    import w4a8_ptq_linear_b200 as oq
    d = 1024
    xb = np.zeros((4, d), np.uint16)
    xb[1] = synth.f64_to_bf16(np.full(d, 0.75))    # constant token
    xb[2] = synth.f64_to_bf16(np.full(d, -3.0))
    xb[3, 5] = synth.f64_to_bf16(np.array([2.0]))[0]   # one non-zero channel
    for center in (False, True):
        plan = oq.Plan(d, 256, 1, center=center, act="int8_absmax")
        codes, scale, mean, _ = oq.rotate_quantize(plan, to_torch_bf16(xb))
        c = codes.cpu().numpy().view(np.int8)
        s = scale.cpu().numpy()
        assert np.all(c[0] == 0) and abs(s[0] - 1e-10 / 127) < 1e-16
        if center:
            # a constant token centers to exactly zero: all codes 0, scale eps / qmax
            m = mean.cpu().numpy()
            assert m[1] == np.float32(0.75) and m[2] == np.float32(-3.0)
            assert np.all(c[1] == 0) and np.all(c[2] == 0)
        plan.close()
    torch.cuda.synchronize()


def test_empty_batch_launches_nothing():
    import torch
    import w4a8_ptq_linear_b200 as oq
    plan = oq.Plan(256, 64, 1)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    codes, scale, _, _ = oq.rotate_quantize(plan, x)
    assert codes.shape == (0, 256)
    plan.close()


def test_row_pitch_larger_than_width():
    import torch
    import w4a8_ptq_linear_b200 as oq
    T, d = 50, 512
    xb = synth.make_x(T, 640, mean_var=1.0, seed=4)
    x = to_torch_bf16(xb)[:, :d]          # ldx = 640
    plan = oq.Plan(d, 128, 2, act="int8_absmax")
    codes, scale, _, _ = oq.rotate_quantize(plan, x)
    codes2, scale2, _, _ = oq.rotate_quantize(plan, x.contiguous())
    assert torch.equal(codes, codes2) and torch.equal(scale, scale2)
    plan.close()


@pytest.mark.parametrize("act", ["int4_percentile", "int2_percentile"])
def test_percentile_clips_outliers_and_handles_flat_tokens(act):
    # CentriQ §4.2: the percentile range leaves the largest magnitudes past +-7 alpha, which
    # clip to +-7; tokens with few distinct magnitudes exercise ties in the order statistics
    import torch
    import w4a8_ptq_linear_b200 as oq
    d, h = 3072, 1024
    xb = synth.make_x(6, d, mean_var=0.0, seed=3)
    x = synth.bf16_to_f64(xb)
    x[0, 17] = 900.0                    # one huge channel
    x[1, :40] = 300.0                   # a block of equal outliers
    x[2] = 0.0                          # zero token
    x[3] = 0.0
    x[3, 5] = 2.0                       # one non-zero channel
    x[4] = np.where(np.arange(d) % 2 == 0, 1.0, -1.0)   # flat magnitudes
    xb = synth.f64_to_bf16(x)
    plan = oq.Plan(d, h, 1, act=act)
    codes, scale, _, rot = oq.rotate_quantize(plan, to_torch_bf16(xb), rotated=True)
    torch.cuda.synchronize()
    ref = oracle.quantize_activations(synth.bf16_to_f64(xb), oracle.rpbh_plan(d, h, 1, 0), h,
                                      act, False)
    qmax = 7 if act == "int4_percentile" else 1
    s = scale.cpu().numpy().astype(np.float64)
    nz = ref["scale"] > 1e-9
    assert np.all(np.abs(s[nz] / ref["scale"][nz] - 1) <= ROT_TOL)
    assert np.all(np.abs(s[~nz] - ref["scale"][~nz]) <= 1e-16)
    gpu = (oracle.unpack_nibbles(codes.cpu().numpy(), signed=True) if qmax == 7
           else oracle.unpack_pairs(codes.cpu().numpy()))
    ex = absmax_boundary_mask(ref["rotated"], ref["scale"], qmax)
    bad, _ = compare_codes(gpu, ref["codes"], ex)
    assert bad == 0
    assert np.abs(gpu[0]).max() == qmax and np.all(gpu[2] == 0)
    plan.close()

