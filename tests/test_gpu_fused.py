"""GPU parity of the single-launch layer (oq_linear_fused) for small token counts, for INT8
absmax and INT4 (absmax, percentile) activations.

The fused kernel runs the same rotate-quantize body and the same integer GEMM arithmetic as the
two-kernel path, with the K dimension split across a cluster of CTAs whose int32 partial sums
are added exactly, and the same epilogue steps. So its output must equal oq_linear's bit for
bit, and its workspace must hold the same codes, scales and means as oq_rotate_quantize's. The
layer is also compared with the oracle at the layer tolerance (8e-3 relative).
"""
import numpy as np
import pytest

import oracle
import synth
from parity import OUT_TOL, rel_fro, to_torch_bf16

pytestmark = pytest.mark.gpu

# (d, n_out, h, rounds, center, bias, T): the DiT width at several token counts (one to 256,
# ragged), the small workload, two rounds with centering and bias, the widest two-token width
CASES = [
    (3072, 3072, 1024, 1, False, False, 1),
    (3072, 3072, 1024, 1, False, False, 2),
    (3072, 3072, 1024, 1, False, False, 77),
    (3072, 3072, 1024, 1, False, False, 256),
    (3072, 3072, 1024, 1, True, True, 131),
    (256, 256, 64, 1, False, False, 64),
    (1920, 1920, 128, 2, True, True, 200),
    (4096, 1024, 256, 2, True, False, 33),
    (8192, 512, 512, 1, False, True, 9),
    (1024, 2048, 16, 1, False, False, 255),
]


def _setup(d, n_out, h, rounds, center, bias, T, seed=0, act="int8_absmax"):
    import w4a8_ptq_linear_b200 as oq
    plan = oq.Plan(d, h, rounds, seed=seed, center=center, act=act)
    xb = synth.make_x(T, d, mean_var=3.0, heavy_frac=0.01, seed=seed + 1)
    wb = synth.make_w(n_out, d, seed=seed)
    bb = synth.make_bias(n_out, seed=seed) if bias else None
    wp, ws, w1 = oq.prepare_weights(plan, to_torch_bf16(wb))
    return plan, xb, wb, bb, wp, ws, w1


@pytest.mark.parametrize("d,n_out,h,rounds,center,bias,T", CASES)
def test_fused_layer_equals_two_kernel_path_and_oracle(d, n_out, h, rounds, center, bias, T):
    import torch
    import w4a8_ptq_linear_b200 as oq
    plan, xb, wb, bb, wp, ws, w1 = _setup(d, n_out, h, rounds, center, bias, T)
    x = to_torch_bf16(xb)
    b = to_torch_bf16(bb) if bb is not None else None
    need = max(plan.workspace_bytes(T), 256)
    ws_f = torch.full((need,), 0xA5, dtype=torch.uint8, device="cuda")
    y_f = oq.linear_fused(plan, x, wp, ws, w1, b, workspace=ws_f)
    y_l = oq.linear(plan, x, wp, ws, w1, b)          # dispatches to the single launch
    codes, scale, mean, _ = oq.rotate_quantize(plan, x)
    y_2 = oq.gemm_w4a8(codes, scale, wp, ws, mean=mean, w_rowsum=w1 if center else None,
                       bias=b)                       # the two-kernel path, call by call
    torch.cuda.synchronize()
    assert torch.equal(y_l, y_f)
    torch.cuda.synchronize()
    st, code = oq.device_status()
    assert st == 0, hex(code)
    assert torch.equal(y_f, y_2), "fused and two-kernel outputs differ"
    # the workspace holds the step's codes, scales and means (oq_linear's layout)
    cb = T * d
    r256 = lambda v: (v + 255) // 256 * 256
    assert torch.equal(ws_f[:cb].view(torch.int8).view(T, d), codes)
    assert torch.equal(ws_f[r256(cb):r256(cb) + 4 * T].view(torch.float32), scale)
    if center:
        off = r256(cb) + r256(4 * T)
        assert torch.equal(ws_f[off:off + 4 * T].view(torch.float32), mean)
    ref, _, _ = oracle.linear_forward(synth.bf16_to_f64(xb), synth.bf16_to_f64(wb),
                                      oracle.rpbh_plan(d, h, rounds, 0), h, "int8_absmax",
                                      center, bias=None if bb is None else synth.bf16_to_f64(bb))
    got = y_f.float().cpu().numpy().astype(np.float64)
    assert rel_fro(got, ref) <= OUT_TOL
    plan.close()


# INT4 codes (absmax, percentile) through the single launch: (d, n_out, h, rounds, center,
# bias, T, act). The DiT width centered and not, one token to 256, two rounds at a narrow
# width, the percentile scale with its clipping, a small block.
CASES_A4 = [
    (3072, 3072, 1024, 1, True, False, 1, "int4_absmax"),
    (3072, 3072, 1024, 1, True, True, 200, "int4_absmax"),
    (3072, 3072, 1024, 1, False, False, 256, "int4_absmax"),
    (1920, 1920, 128, 2, True, False, 37, "int4_absmax"),
    (3072, 3072, 1024, 1, True, False, 64, "int4_percentile"),
    (1024, 2048, 16, 1, False, True, 255, "int4_percentile"),
]


@pytest.mark.parametrize("d,n_out,h,rounds,center,bias,T,act", CASES_A4)
def test_fused_int4_layer_equals_two_kernel_path_and_oracle(d, n_out, h, rounds, center, bias,
                                                             T, act):
    # The single launch multiplies the INT4 codes, stored one byte each, with the kind::i8
    # GEMM; the two kernels pack them two per byte and widen both operands. The integer sums
    # differ only by a power of two that the epilogue's scale undoes exactly, so the outputs
    # agree bit for bit.
    import torch
    import w4a8_ptq_linear_b200 as oq
    plan, xb, wb, bb, wp, ws, w1 = _setup(d, n_out, h, rounds, center, bias, T, act=act)
    x = to_torch_bf16(xb)
    b = to_torch_bf16(bb) if bb is not None else None
    need = max(plan.workspace_bytes(T), 256)
    assert need >= T * d   # one byte per code where the single launch may run
    ws_f = torch.full((need,), 0xA5, dtype=torch.uint8, device="cuda")
    y_f = oq.linear_fused(plan, x, wp, ws, w1, b, workspace=ws_f)
    y_l = oq.linear(plan, x, wp, ws, w1, b)          # dispatches to the single launch
    codes, scale, mean, _ = oq.rotate_quantize(plan, x)
    y_2 = oq.gemm_w4a4(plan, act, codes, scale, wp, ws, mean=mean,
                       w_rowsum=w1 if center else None, bias=b)   # the two kernels
    torch.cuda.synchronize()
    st, code = oq.device_status()
    assert st == 0, hex(code)
    assert torch.equal(y_l, y_f)
    assert torch.equal(y_f, y_2), "fused and two-kernel outputs differ"
    # the workspace: the same codes one byte each, the same scales and means
    cb = T * d
    r256 = lambda v: (v + 255) // 256 * 256
    got_codes = ws_f[:cb].view(torch.int8).view(T, d).cpu().numpy()
    want_codes = oracle.unpack_nibbles(codes.cpu().numpy(), signed=True)
    np.testing.assert_array_equal(got_codes.astype(np.int64), want_codes.astype(np.int64))
    assert np.abs(got_codes).max() <= 7
    assert torch.equal(ws_f[r256(cb):r256(cb) + 4 * T].view(torch.float32), scale)
    if center:
        off = r256(cb) + r256(4 * T)
        assert torch.equal(ws_f[off:off + 4 * T].view(torch.float32), mean)
    ref, _, _ = oracle.linear_forward(synth.bf16_to_f64(xb), synth.bf16_to_f64(wb),
                                      oracle.rpbh_plan(d, h, rounds, 0), h, act, center,
                                      bias=None if bb is None else synth.bf16_to_f64(bb))
    got = y_f.float().cpu().numpy().astype(np.float64)
    assert rel_fro(got, ref) <= OUT_TOL
    plan.close()


def test_fused_layer_repeated_calls_are_identical():
    # the grid barrier and the cluster exchange leave nothing behind between launches
    import torch
    import w4a8_ptq_linear_b200 as oq
    plan, xb, wb, bb, wp, ws, w1 = _setup(3072, 3072, 1024, 1, False, False, 200)
    x = to_torch_bf16(xb)
    ys = [oq.linear_fused(plan, x, wp, ws, w1) for _ in range(20)]
    torch.cuda.synchronize()
    assert oq.device_status()[0] == 0
    assert all(torch.equal(ys[0], y) for y in ys[1:])
    plan.close()


def test_fused_layer_rejects_what_it_does_not_cover():
    import torch
    import w4a8_ptq_linear_b200 as oq
    plan, xb, wb, bb, wp, ws, w1 = _setup(256, 256, 64, 1, False, False, 257)
    x = to_torch_bf16(xb)
    with pytest.raises(oq.OQError) as e:
        oq.linear_fused(plan, x, wp, ws, w1)
    assert e.value.status == oq.OQ_ERR_UNSUPPORTED
    plan.close()
    for act in ("int2_percentile", "int4_lloydmax", "int8_lloydmax"):
        pk = oq.Plan(256, 64, 1, act=act)
        with pytest.raises(oq.OQError) as e:
            oq.linear_fused(pk, x[:8], wp, ws, w1)
        assert e.value.status == oq.OQ_ERR_UNSUPPORTED
        pk.close()
    torch.cuda.synchronize()
    assert oq.device_status()[0] == 0
