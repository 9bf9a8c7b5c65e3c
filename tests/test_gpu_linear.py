"""GPU parity of the whole layer (oq_prepare_weights + oq_linear) against the oracle.

Per workload: a reduced token count that spans several tiles with a ragged tail is checked on
every output; the full-size workload, in the launch configuration the benchmark times, is
checked on a seeded sample of token rows (tokens are independent, so those rows are exact
parity). Final bf16 outputs: <= 8e-3 relative (Frobenius).
"""
import numpy as np
import pytest

import oracle
import synth
from parity import OUT_TOL, rel_fro, to_torch_bf16

pytestmark = pytest.mark.gpu


def _oracle_rows(wl, xb_rows, wb, bias=None):
    c, t = (oracle.lloyd_max_sphere(wl.d) if wl.act == "int4_lloydmax_width"
            else oracle.lloyd_max_gaussian_8bit() if wl.act == "int8_lloydmax"
            else oracle.lloyd_max_gaussian())
    plan = oracle.rpbh_plan(wl.d, wl.h, wl.rounds, wl.seed)
    y, _, _ = oracle.linear_forward(synth.bf16_to_f64(xb_rows), synth.bf16_to_f64(wb), plan,
                                    wl.h, wl.act, wl.center, bias=bias, centroids=c,
                                    thresholds=t)
    return y


def _gpu_layer(wl, xb, wb, bias_bits=None):
    import torch
    import w4a8_ptq_linear_b200 as oq
    plan = oq.Plan(wl.d, wl.h, wl.rounds, seed=wl.seed, center=wl.center, act=wl.act)
    wp, ws, w1 = oq.prepare_weights(plan, to_torch_bf16(wb))
    bias = to_torch_bf16(bias_bits) if bias_bits is not None else None
    y = oq.linear(plan, to_torch_bf16(xb), wp, ws, w1, bias)
    torch.cuda.synchronize()
    st, code = oq.device_status()
    assert st == 0, hex(code)
    out = y.float().cpu().numpy().astype(np.float64)
    plan.close()
    return out


@pytest.mark.parametrize("name,T", [("tiny", 64), ("dit_w4a8", 300), ("dit_lm8", 300),
                                    ("narrow_lm", 257),
                                    ("narrow_lm_w", 257), ("mlp_up", 130), ("mlp_up_pct", 130),
                                    ("mlp_up_a2", 130), ("mlp_up_a2", 1)])
def test_layer_matches_oracle(name, T):
    wl, xb, wb = synth.make_inputs(name, T=T)
    y = _gpu_layer(wl, xb, wb)
    ref = _oracle_rows(wl, xb, wb)
    assert rel_fro(y, ref) <= OUT_TOL


def test_layer_with_bias():
    wl, xb, wb = synth.make_inputs("mlp_up", T=70)
    bias = synth.make_bias(wl.n_out, seed=9)
    y = _gpu_layer(wl, xb, wb, bias)
    ref = _oracle_rows(wl, xb, wb, bias=synth.bf16_to_f64(bias))
    assert rel_fro(y, ref) <= OUT_TOL


@pytest.mark.parametrize("name", ["dit_w4a8", "dit_lm8", "narrow_lm", "narrow_lm_w", "mlp_up",
                                  "mlp_up_pct", "mlp_up_a2"])
def test_full_size_layer_on_sampled_rows(name):
    wl, xb, wb = synth.make_inputs(name)
    y = _gpu_layer(wl, xb, wb)
    rows = np.sort(np.random.default_rng(42).choice(wl.T, 48, replace=False))
    rows = np.unique(np.concatenate([rows, [0, wl.T - 1]]))
    ref = _oracle_rows(wl, xb[rows], wb)
    assert rel_fro(y[rows], ref) <= OUT_TOL
    assert np.all(np.isfinite(y))


def test_linear_equals_separate_calls():
    import torch
    import w4a8_ptq_linear_b200 as oq
    wl, xb, wb = synth.make_inputs("mlp_up", T=200)
    plan = oq.Plan(wl.d, wl.h, wl.rounds, center=True, act=wl.act)
    wp, ws, w1 = oq.prepare_weights(plan, to_torch_bf16(wb))
    x = to_torch_bf16(xb)
    y1 = oq.linear(plan, x, wp, ws, w1)
    codes, scale, mean, _ = oq.rotate_quantize(plan, x)
    y2 = oq.gemm_w4a4(plan, wl.act, codes, scale, wp, ws, mean=mean, w_rowsum=w1)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    plan.close()


def test_offset_invariance_on_gpu():
    # CentriQ Eq. 6: centered codes and scales do not change when c * 1 is added to a token;
    # x on a coarse grid and c = 0.375 keep the bf16 inputs and their sums exact.
    import torch
    import w4a8_ptq_linear_b200 as oq
    rng = np.random.default_rng(0)
    x = np.round(rng.standard_normal((96, 1024)) * 8) / 8
    plan = oq.Plan(1024, 1024, 1, center=True, act="int4_absmax")
    c1, s1, m1, _ = oq.rotate_quantize(plan, to_torch_bf16(synth.f64_to_bf16(x)))
    c2, s2, m2, _ = oq.rotate_quantize(plan, to_torch_bf16(synth.f64_to_bf16(x + 0.375)))
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(s1, s2)
    assert torch.allclose(m2 - m1, torch.full_like(m1, 0.375), atol=1e-6)
    plan.close()
