"""GPU parity of the fused center + RPBH + quantize kernel at the sweep's full token count.

The bandwidth sweep runs T = 65536 tokens. At that count every persistent CTA makes hundreds
of passes: the two-token kernel (d <= 8192) cycles its landing buffer, and the single-token
kernel (d = 30720) wraps its look-ahead ring many times. Tokens are independent (one scale per
token, CentriQ Eq. 1), so the oracle checks a seeded sample of 512 rows plus the first and last
two. On those rows the comparison is the same as for small T: rotated values within 1e-5
relative per token, scales within 1e-5, and codes identical except within 1e-5 relative of a
decision boundary.
"""
import numpy as np
import pytest

import oracle
import synth
from parity import (ROT_TOL, absmax_boundary_mask, compare_codes, lloyd_max_boundary_mask,
                    per_token_rel, to_torch_bf16)

pytestmark = pytest.mark.gpu

T_FULL = 65536
N_SAMPLE = 512

# (d, h, rounds, act): the widest width at the smallest and largest block, and the two-token
# kernel at block sizes other than the layer workloads' (h = 1024 one round, h = 128 two rounds)
CASES = [(30720, h, r, act) for h in (64, 1024) for r in (1, 2)
         for act in ("int8_absmax", "int4_lloydmax")]
CASES += [(1920, 64, r, act) for r in (1, 2) for act in ("int8_absmax", "int4_lloydmax")]
CASES += [(4096, h, r, act) for h in (64, 256) for r in (1, 2)
          for act in ("int8_absmax", "int4_lloydmax")]
CASES += [(3072, 1024, 1, "int8_absmax"), (3072, 512, 2, "int4_lloydmax")]

_X = {}


def _x_device(d):
    """The sweep's activations at width d (as the bench draws them), on the host and the GPU;
    one width at a time stays resident."""
    if d not in _X:
        _X.clear()
        xb = synth.make_x_parallel(T_FULL, d, mean_var=3.0, heavy_frac=0.01, seed=0)
        _X[d] = (xb, to_torch_bf16(xb))
    return _X[d]


def _rows():
    rng = np.random.default_rng(2024)
    rows = rng.choice(T_FULL, N_SAMPLE, replace=False)
    return np.unique(np.concatenate([rows, [0, 1, T_FULL - 2, T_FULL - 1]]))


@pytest.mark.parametrize("d,h,rounds,act", CASES)
def test_full_sweep_size_on_sampled_rows(d, h, rounds, act):
    import torch
    import w4a8_ptq_linear_b200 as oq
    xb, x = _x_device(d)
    plan = oq.Plan(d, h, rounds, seed=0, center=False, act=act)
    codes, scale, _, rot = oq.rotate_quantize(plan, x, rotated=True)
    torch.cuda.synchronize()
    st, code = oq.device_status()
    assert st == 0, hex(code)
    rows = _rows()
    idx = torch.from_numpy(rows).cuda()
    g_codes = codes.index_select(0, idx).cpu().numpy()
    g_scale = scale.index_select(0, idx).cpu().numpy().astype(np.float64)
    g_rot = rot.index_select(0, idx).cpu().numpy().astype(np.float64)
    del codes, scale, rot
    plan.close()
    thresholds = oracle.lloyd_max_gaussian()[1]
    ref = oracle.quantize_activations(synth.bf16_to_f64(xb[rows]),
                                      oracle.rpbh_plan(d, h, rounds, 0), h, act, False,
                                      thresholds)
    assert per_token_rel(g_rot, ref["rotated"]).max() <= ROT_TOL
    assert np.abs(g_scale / ref["scale"] - 1).max() <= ROT_TOL
    if act == "int8_absmax":
        gpu = g_codes.view(np.int8).astype(np.int64)
        ex = absmax_boundary_mask(ref["rotated"], ref["scale"], 127)
    else:
        gpu = oracle.unpack_nibbles(g_codes, signed=False)
        ex = lloyd_max_boundary_mask(ref["rotated"], ref["scale"], thresholds)
    bad, n_ex = compare_codes(gpu, ref["codes"], ex)
    assert bad == 0, f"{bad} codes differ outside the boundary exemption ({n_ex} exempt)"
