"""The allocation-free entry point oq_linear_static_scratch, through the C ABI.

Some callers cannot allocate device scratch: plug-ins inside a framework that owns all device
memory, or paths that may not call cudaMalloc. For them the library keeps its own fixed
scratch array. This file checks that the entry point gives bit for bit the layer output of
oq_linear with a caller-owned workspace (the same kernels on the same inputs, only the scratch
pointer differs) on three calls in a row, each with fewer tokens than the one before, so that
a call's scales and means sit where the previous call left codes: it must not be disturbed by
what the earlier calls left in the shared array. It also checks that the entry point
refuses a batch too large for the array. It is collected last so that a failure here comes
after every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from parity import to_torch_bf16

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 16 << 20


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("name", ["dit_w4a8", "mlp_up"])
def test_static_scratch_matches_linear_on_consecutive_calls(name):
    import w4a8_ptq_linear_b200 as oq
    L = oq.lib()
    wl = synth.WORKLOADS[name]
    plan = oq.Plan(wl.d, wl.h, wl.rounds, seed=wl.seed, center=wl.center, act=wl.act)
    wp, ws, w1 = oq.prepare_weights(plan, to_torch_bf16(synth.make_w(wl.n_out, wl.d)))
    w1 = w1 if wl.center else None
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # two calls in a row, different tokens; the first is larger, so the regions of the shared
    # array that hold the second call's scales and means move
    # (a third call of 100 tokens takes the single-launch path for the DiT plan; the MLP-up
    # layer's 96 channel tiles do not fit on the device at once, so it takes the two kernels)
    for call, (T, seed) in enumerate(((2000, 11), (777, 12), (100, 13))):
        assert plan.workspace_bytes(T) <= STATIC_SCRATCH_BYTES
        xb = synth.make_x(T, wl.d, mean_var=wl.mean_var, heavy_frac=wl.heavy_frac, seed=seed)
        x = to_torch_bf16(xb)
        y_ref = oq.linear(plan, x, wp, ws, w1)      # caller-owned workspace
        y = torch.full_like(y_ref, float("nan"))
        st = L.oq_linear_static_scratch(plan.handle, _p(x), T, x.stride(0), _p(wp), _p(ws),
                                        _p(w1), None, wl.n_out, _p(y), stream)
        assert st == 0, L.oq_last_error()
        torch.cuda.synchronize()
        assert oq.device_status()[0] == 0
        assert torch.equal(y, y_ref), f"call {call}: outputs differ"
        got = y.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), f"call {call}"
    plan.close()


def test_static_scratch_rejects_too_many_tokens():
    import w4a8_ptq_linear_b200 as oq
    L = oq.lib()
    plan = oq.Plan(3072, 1024, 1, act="int8_absmax")
    T = 5448                                        # first T whose scratch exceeds 16 MiB
    assert plan.workspace_bytes(T) > STATIC_SCRATCH_BYTES >= plan.workspace_bytes(T - 1)
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    st = L.oq_linear_static_scratch(plan.handle, _p(dummy), T, 3072, _p(dummy), _p(dummy), None,
                                    None, 3072, _p(dummy), None)
    assert st == oq.OQ_ERR_INVALID_ARG
    assert b"static" in L.oq_last_error()
    plan.close()
