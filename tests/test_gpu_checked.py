"""The bounds-checked build (-DOQ_CHECKED) on the GPU.

In the checked build every table-driven device index (the rotation's gathers and the
interleave's word offsets, the round-2 buffer, the single-launch layer's ring stages, partial
sums and token shares) is range-checked, and a violation is reported through the device error
word as OQ_ERR_INVALID_ARG instead of touching memory. Each case runs the same call through the
checked and the release library on the same inputs: the checked run must report nothing and
return the same bits.
"""
import pytest

import synth
from parity import to_torch_bf16

pytestmark = pytest.mark.gpu

# (T, d, h, rounds, act, center): the two-token kernel (both rounds, every transform shape),
# the single-token kernel, the percentile and 2-bit quantizers
RQ_CASES = [
    (33, 3072, 1024, 2, "int8_absmax", True),
    (9, 1920, 64, 2, "int4_lloydmax", False),
    (7, 256, 1, 1, "int4_absmax", False),
    (45, 4096, 256, 1, "int2_percentile", True),
    (5, 30720, 1024, 2, "int8_absmax", True),
    (4, 30720, 32, 1, "int4_lloydmax", False),
]


def _both(fn):
    """fn() run against the release build, then against the checked build."""
    import torch
    import w4a8_ptq_linear_b200 as oq
    out = fn()
    torch.cuda.synchronize()
    assert oq.device_status()[0] == 0
    with oq.using(oq.load(oq.LIB_CHECKED_PATH)):
        out_c = fn()
        torch.cuda.synchronize()
        st, code = oq.device_status()
        assert st == 0, f"checked build reported {code:#x}"
    return out, out_c


@pytest.mark.parametrize("T,d,h,rounds,act,center", RQ_CASES)
def test_checked_rotate_quantize_is_clean_and_identical(T, d, h, rounds, act, center):
    import torch
    import w4a8_ptq_linear_b200 as oq
    x = to_torch_bf16(synth.make_x(T, d, mean_var=3.0, heavy_frac=0.01, seed=3))

    def run():
        plan = oq.Plan(d, h, rounds, center=center, act=act)
        codes, scale, mean, rot = oq.rotate_quantize(plan, x, rotated=True)
        plan.close()
        return codes, scale, mean, rot

    a, b = _both(run)
    for u, v in zip(a, b):
        assert (u is None and v is None) or torch.equal(u, v)


@pytest.mark.parametrize("name,T", [("dit_w4a8", 77), ("dit_w4a8", 300), ("mlp_up_a2", 130)])
def test_checked_layer_is_clean_and_identical(name, T):
    import torch
    import w4a8_ptq_linear_b200 as oq
    wl, xb, wb = synth.make_inputs(name, T=T)
    x, w = to_torch_bf16(xb), to_torch_bf16(wb)

    def run():
        plan = oq.Plan(wl.d, wl.h, wl.rounds, seed=wl.seed, center=wl.center, act=wl.act)
        wp, ws, w1 = oq.prepare_weights(plan, w)
        y = oq.linear(plan, x, wp, ws, w1 if wl.center else None)
        plan.close()
        return y

    y, y_c = _both(run)
    assert torch.equal(y, y_c)
