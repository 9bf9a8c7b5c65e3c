"""Error paths on the GPU: argument checks return a status before any launch, and a bounded
device-side wait that can never complete gives up, records a timeout and leaves the context
usable (no trap, no fault, no hang)."""
import numpy as np
import pytest
import torch

import synth
from parity import to_torch_bf16

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_survives():
    import w4a8_ptq_linear_b200 as oq
    oq.device_status(clear=True)
    oq.debug_wait_timeout(50_000_000)           # 50 ms; nothing ever arrives
    st, code = oq.device_status(clear=True)
    assert st == oq.OQ_ERR_DEVICE_TIMEOUT
    assert (code >> 63) == 1 and ((code >> 32) & 0xFFFF) == 99
    assert oq.device_status()[0] == 0            # cleared
    # the device still computes correctly afterwards
    plan = oq.Plan(256, 64, 1)
    xb = synth.make_x(8, 256, mean_var=1.0)
    codes, scale, _, _ = oq.rotate_quantize(plan, to_torch_bf16(xb))
    torch.cuda.synchronize()
    assert torch.isfinite(scale).all()
    plan.close()


def test_misaligned_and_invalid_arguments():
    import w4a8_ptq_linear_b200 as oq
    plan = oq.Plan(256, 64, 1)
    x = torch.zeros((4, 264), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(oq.OQError) as e:
        oq.rotate_quantize(plan, x[:, 1:257])    # base not 16-byte aligned
    assert e.value.status == oq.OQ_ERR_MISALIGNED
    wp = torch.zeros((100, 128), dtype=torch.uint8, device="cuda")
    ws = torch.ones(100, dtype=torch.float32, device="cuda")
    a = torch.zeros((4, 256), dtype=torch.int8, device="cuda")
    with pytest.raises(oq.OQError) as e:
        oq.gemm_w4a8(a, ws[:4], wp, ws)          # d_out = 100 is not a multiple of 16
    assert e.value.status == oq.OQ_ERR_INVALID_ARG
    with pytest.raises(oq.OQError):
        oq.gemm_w4a4(None, "int4_lloydmax", wp[:4], ws[:4], wp[:96], ws[:96])  # no codebook
    plan.close()
    assert oq.device_status()[0] == 0


def test_plan_rejects_other_device_or_bad_shape():
    import w4a8_ptq_linear_b200 as oq
    with pytest.raises(oq.OQError):
        oq.Plan(3072, 2048, 1)
    p = oq.Plan(3072, 1024, 1, seed=5, center=True, act="int4_absmax")
    s, perm = p.rpbh(0)
    s2, perm2 = oq.rpbh_tables(3072, 0, 5)
    assert np.array_equal(s, s2) and np.array_equal(perm, perm2)
    p.close()


@pytest.mark.parametrize("act,d,levels", [("int4_lloydmax", 1920, 16),
                                          ("int4_lloydmax_width", 1920, 16),
                                          ("int4_lloydmax_width", 256, 16),
                                          ("int8_lloydmax", 3072, 256)])
def test_plan_codebook_is_the_oracle_table(act, d, levels):
    # oq_plan_get_codebook returns the table the plan quantizes with; the oracle solves the
    # same optimality conditions by Lloyd iteration (the library by Newton's method)
    import oracle
    import w4a8_ptq_linear_b200 as oq
    p = oq.Plan(d, 128 if d % 128 == 0 else 64, 1, act=act)
    c, t = p.codebook()
    ref_c, ref_t = (oracle.lloyd_max_sphere(d) if act == "int4_lloydmax_width"
                    else oracle.lloyd_max_gaussian_8bit() if levels == 256
                    else oracle.lloyd_max_gaussian())
    assert c.shape == (levels,) and t.shape == (levels - 1,)
    assert np.abs(c - ref_c).max() < 1e-8 and np.abs(t - ref_t).max() < 1e-8
    assert np.all(np.diff(c) > 0) and np.allclose(t, (c[1:] + c[:-1]) / 2, rtol=0, atol=1e-12)
    # a wrong level count and a plan without a codebook are argument errors
    wrong = np.empty(256 if levels == 16 else 16)
    with pytest.raises(oq.OQError) as e:
        oq._check(oq.lib().oq_plan_get_codebook(p.handle, wrong.size, wrong.ctypes.data,
                                                wrong.ctypes.data))
    assert e.value.status == oq.OQ_ERR_INVALID_ARG
    p.close()
    q = oq.Plan(256, 64, 1, act="int8_absmax")
    with pytest.raises(oq.OQError) as e:
        q.codebook()
    assert e.value.status == oq.OQ_ERR_INVALID_ARG
    q.close()
