"""GPU parity of the tcgen05 GEMMs and their epilogue, and of the weight preparation.

Integer GEMMs are fed the oracle's codes and must return bit-exact int32 accumulators.
The Lloyd-Max GEMM decodes codes to fp16 centroids: its fp32 accumulators are compared with
the oracle's fp64 sum over the same fp16-rounded centroids (the GEMM arithmetic itself) and
with the exact centroids (the layer's tolerance). The fused epilogue is compared with the
oracle's epilogue at 8e-3 relative.
"""
import numpy as np
import pytest

import oracle
import synth
from parity import (OUT_TOL, absmax_boundary_mask, compare_codes, pack_w4_gemm, rel_fro,
                    to_torch_bf16, unpack_w4_gemm)

pytestmark = pytest.mark.gpu

SHAPES = [(64, 256, 256), (200, 384, 272), (513, 3072, 3072), (129, 1920, 1920),
          (7, 128, 16), (300, 256, 4096),
          # 100 CTA-pair tiles: more than one wave of pairs on a 148-SM part
          (2560, 1536, 2560)]


def _codes(rng, T, K, N, amax):
    a = rng.integers(-amax, amax + 1, (T, K))
    w = rng.integers(-7, 8, (N, K))
    # make some rows extreme so the int32 range is exercised
    a[0, :] = amax
    w[0, :] = 7
    return a, w


@pytest.mark.parametrize("T,K,N", SHAPES)
def test_w4a8_accumulators_bit_exact(T, K, N):
    import torch
    import w4a8_ptq_linear_b200 as oq
    rng = np.random.default_rng(T + K + N)
    a, w = _codes(rng, T, K, N, 127)
    at = torch.from_numpy(a.astype(np.int8)).cuda()
    wp = torch.from_numpy(pack_w4_gemm(w)).cuda()
    ones = torch.ones(max(T, N), dtype=torch.float32, device="cuda")
    acc = oq.gemm_w4a8(at, ones[:T], wp, ones[:N], out_kind=oq.OUT_ACC)
    torch.cuda.synchronize()
    assert oq.device_status()[0] == 0
    ref = oracle.gemm_int(a, w).astype(np.int64)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref)


@pytest.mark.parametrize("T,K,N", SHAPES)
def test_w4a4_absmax_accumulators_bit_exact(T, K, N):
    import torch
    import w4a8_ptq_linear_b200 as oq
    rng = np.random.default_rng(7 * T + K + N)
    a, w = _codes(rng, T, K, N, 7)
    ap = torch.from_numpy(oracle.pack_nibbles(a)).cuda()
    wp = torch.from_numpy(pack_w4_gemm(w)).cuda()
    ones = torch.ones(max(T, N), dtype=torch.float32, device="cuda")
    acc = oq.gemm_w4a4(None, "int4_absmax", ap, ones[:T], wp, ones[:N], out_kind=oq.OUT_ACC)
    torch.cuda.synchronize()
    ref = oracle.gemm_int(a, w).astype(np.int64)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref)


@pytest.mark.parametrize("T,K,N", SHAPES)
def test_w4a2_accumulators_bit_exact(T, K, N):
    import torch
    import w4a8_ptq_linear_b200 as oq
    rng = np.random.default_rng(5 * T + K + N)
    a, w = _codes(rng, T, K, N, 1)
    a[1, :] = -1
    w[1, :] = -7
    ap = torch.from_numpy(oracle.pack_pairs(a)).cuda()
    wp = torch.from_numpy(pack_w4_gemm(w)).cuda()
    ones = torch.ones(max(T, N), dtype=torch.float32, device="cuda")
    acc = oq.gemm_w4a2(ap, ones[:T], wp, ones[:N], out_kind=oq.OUT_ACC)
    torch.cuda.synchronize()
    assert oq.device_status()[0] == 0
    ref = oracle.gemm_int(a, w).astype(np.int64)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref)


def test_w4a2_rejects_width_not_multiple_of_64():
    import torch
    import w4a8_ptq_linear_b200 as oq
    ap = torch.zeros((8, 24), dtype=torch.uint8, device="cuda")     # K = 96
    wp = torch.zeros((16, 48), dtype=torch.uint8, device="cuda")
    ones = torch.ones(16, dtype=torch.float32, device="cuda")
    with pytest.raises(oq.OQError) as e:
        oq.gemm_w4a2(ap, ones[:8], wp, ones, out_kind=oq.OUT_ACC)
    assert e.value.status == oq.OQ_ERR_INVALID_ARG


@pytest.mark.parametrize("T,K,N", [(64, 256, 256), (200, 384, 272), (130, 1920, 1920),
                                   (2560, 1536, 2560)])
def test_lloyd_max_accumulators(T, K, N):
    import torch
    import w4a8_ptq_linear_b200 as oq
    rng = np.random.default_rng(3 * T + K)
    codes = rng.integers(0, 16, (T, K))
    w = rng.integers(-7, 8, (N, K))
    plan = oq.Plan(K, 64, 1, act="int4_lloydmax")
    ap = torch.from_numpy(oracle.pack_nibbles(codes)).cuda()
    wp = torch.from_numpy(pack_w4_gemm(w)).cuda()
    ones = torch.ones(max(T, N), dtype=torch.float32, device="cuda")
    acc = oq.gemm_w4a4(plan, "int4_lloydmax", ap, ones[:T], wp, ones[:N], out_kind=oq.OUT_ACC)
    acc = acc.cpu().numpy().astype(np.float64)
    c, _ = oracle.lloyd_max_gaussian()
    c16 = c.astype(np.float16).astype(np.float64)
    # same decoded centroids: only fp32 accumulation order differs
    assert rel_fro(acc, oracle.gemm_lloyd_max(codes, c16, w)) < 1e-6
    # exact centroids: the fp16 decode stays far inside the layer's output tolerance
    assert rel_fro(acc, oracle.gemm_lloyd_max(codes, c, w)) < 1e-3
    plan.close()


@pytest.mark.parametrize("kind", ["int8_absmax", "int4_absmax", "int4_lloydmax",
                                  "int2_percentile"])
@pytest.mark.parametrize("with_mean,with_bias", [(False, False), (True, True), (True, False)])
def test_epilogue_matches_oracle(kind, with_mean, with_bias):
    import torch
    import w4a8_ptq_linear_b200 as oq
    T, K, N = 260, 512, 384
    rng = np.random.default_rng(11)
    amax = {"int8_absmax": 127, "int2_percentile": 1}.get(kind, 7)
    if kind == "int4_lloydmax":
        a = rng.integers(0, 16, (T, K))
    else:
        a = rng.integers(-amax, amax + 1, (T, K))
    w = rng.integers(-7, 8, (N, K))
    scale = rng.uniform(0.001, 0.1, T).astype(np.float32)
    s_w = rng.uniform(0.001, 0.05, N).astype(np.float32)
    mean = rng.normal(0, 3, T).astype(np.float32)
    w1 = rng.normal(0, 1, N).astype(np.float32)
    bias_bits = synth.make_bias(N, seed=2)
    plan = oq.Plan(K, 64, 1, act=kind)
    cuda = lambda v: torch.from_numpy(v).cuda()
    mean_t = cuda(mean) if with_mean else None
    w1_t = cuda(w1) if with_mean else None
    bias_t = to_torch_bf16(bias_bits) if with_bias else None
    wp = cuda(pack_w4_gemm(w))
    if kind == "int8_absmax":
        y = oq.gemm_w4a8(cuda(a.astype(np.int8)), cuda(scale), wp, cuda(s_w), mean=mean_t,
                         w_rowsum=w1_t, bias=bias_t)
        acc = oracle.gemm_int(a, w)
    elif kind == "int2_percentile":
        y = oq.gemm_w4a2(cuda(oracle.pack_pairs(a)), cuda(scale), wp, cuda(s_w), mean=mean_t,
                         w_rowsum=w1_t, bias=bias_t)
        acc = oracle.gemm_int(a, w)
    else:
        y = oq.gemm_w4a4(plan, kind, cuda(oracle.pack_nibbles(a)), cuda(scale), wp, cuda(s_w),
                         mean=mean_t, w_rowsum=w1_t, bias=bias_t)
        acc = (oracle.gemm_int(a, w) if kind == "int4_absmax"
               else oracle.gemm_lloyd_max(a, oracle.lloyd_max_gaussian()[0], w))
    ref = oracle.epilogue(acc, scale.astype(np.float64), s_w.astype(np.float64),
                          mean.astype(np.float64) if with_mean else None,
                          w1.astype(np.float64) if with_mean else None,
                          synth.bf16_to_f64(bias_bits) if with_bias else None)
    got = y.float().cpu().numpy().astype(np.float64)
    assert rel_fro(got, ref) <= OUT_TOL
    # bf16 rounding is the dominant difference: stays near 2^-9 per element
    assert rel_fro(got, ref) < 3e-3
    plan.close()


@pytest.mark.parametrize("n_out,d,h,rounds", [(256, 256, 64, 1), (3072, 3072, 1024, 1),
                                              (1920, 1920, 128, 2), (48, 4096, 512, 1)])
def test_prepare_weights_matches_oracle(n_out, d, h, rounds):
    import torch
    import w4a8_ptq_linear_b200 as oq
    wb = synth.make_w(n_out, d, seed=5)
    plan = oq.Plan(d, h, rounds)
    wp, ws, w1 = oq.prepare_weights(plan, to_torch_bf16(wb))
    torch.cuda.synchronize()
    w = synth.bf16_to_f64(wb)
    op = oracle.rpbh_plan(d, h, rounds, 0)
    codes, s_w, w1_ref = oracle.prepare_weights(w, op, h)
    assert np.abs(ws.cpu().numpy() / s_w - 1).max() <= 1e-5
    assert np.all(np.abs(w1.cpu().numpy() - w1_ref) <= 1e-5 * np.abs(w).sum(axis=1))
    gpu = unpack_w4_gemm(wp.cpu().numpy())
    ex = absmax_boundary_mask(oracle.rotate(w, op, h), s_w, 7)
    bad, _ = compare_codes(gpu, codes, ex)
    assert bad == 0
    plan.close()


@pytest.mark.parametrize("T,K,N", [(64, 256, 256), (200, 384, 272), (300, 3072, 3072),
                                   (2560, 1536, 2560)])
def test_lloyd_max_8bit_accumulators_and_epilogue(T, K, N):
    import torch
    import w4a8_ptq_linear_b200 as oq
    rng = np.random.default_rng(5 * T + K)
    codes = rng.integers(0, 256, (T, K))
    w = rng.integers(-7, 8, (N, K))
    plan = oq.Plan(K, 64, 1, act="int8_lloydmax")
    cu = lambda v: torch.from_numpy(np.ascontiguousarray(v)).cuda()
    ap, wp = cu(codes.astype(np.uint8)), cu(pack_w4_gemm(w))
    ones = torch.ones(max(T, N), dtype=torch.float32, device="cuda")
    acc = oq.gemm_w4a8_lloydmax(plan, ap, ones[:T], wp, ones[:N], out_kind=oq.OUT_ACC)
    acc = acc.cpu().numpy().astype(np.float64)
    c, _ = oq.lloyd_max_codebook_8bit()
    c16 = c.astype(np.float16).astype(np.float64)
    # the same fp16 centroids: only the fp32 accumulation order differs
    assert rel_fro(acc, oracle.gemm_lloyd_max(codes, c16, w)) < 1e-6
    c_or, _ = oracle.lloyd_max_gaussian_8bit()
    assert rel_fro(acc, oracle.gemm_lloyd_max(codes, c_or, w)) < 1e-3
    # epilogue with scales, rank-1 term and bias
    scale = rng.uniform(0.001, 0.1, T).astype(np.float32)
    s_w = rng.uniform(0.001, 0.05, N).astype(np.float32)
    mean = rng.normal(0, 3, T).astype(np.float32)
    w1 = rng.normal(0, 1, N).astype(np.float32)
    bias_bits = synth.make_bias(N, seed=4)
    y = oq.gemm_w4a8_lloydmax(plan, ap, cu(scale), wp, cu(s_w), mean=cu(mean), w_rowsum=cu(w1),
                              bias=to_torch_bf16(bias_bits))
    ref = oracle.epilogue(oracle.gemm_lloyd_max(codes, c_or, w), scale.astype(np.float64),
                          s_w.astype(np.float64), mean.astype(np.float64), w1.astype(np.float64),
                          synth.bf16_to_f64(bias_bits))
    assert rel_fro(y.float().cpu().numpy().astype(np.float64), ref) <= OUT_TOL
    plan.close()



@pytest.mark.parametrize("T", [1, 37, 128, 200, 256])
@pytest.mark.parametrize("with_mean,with_bias", [(False, False), (True, True)])
def test_small_t_w4a8_split_k_matches_oracle(T, with_mean, with_bias):
    # up to 256 tokens the W4A8 GEMM with a bf16 result runs split-K over clusters, the int32
    # partial sums added through distributed shared memory; the result is compared with the
    # oracle's epilogue on the same codes, and with the same call one token at a time
    import torch
    import w4a8_ptq_linear_b200 as oq
    K, N = 3072, 3072
    rng = np.random.default_rng(100 + T)
    a = rng.integers(-127, 128, (T, K))
    w = rng.integers(-7, 8, (N, K))
    scale = rng.uniform(0.001, 0.1, T).astype(np.float32)
    s_w = rng.uniform(0.001, 0.05, N).astype(np.float32)
    mean = rng.normal(0, 3, T).astype(np.float32)
    w1 = rng.normal(0, 1, N).astype(np.float32)
    bias_bits = synth.make_bias(N, seed=4)
    cuda = lambda v: torch.from_numpy(v).cuda()
    mean_t = cuda(mean) if with_mean else None
    w1_t = cuda(w1) if with_mean else None
    bias_t = to_torch_bf16(bias_bits) if with_bias else None
    at, wp = cuda(a.astype(np.int8)), cuda(pack_w4_gemm(w))
    y = oq.gemm_w4a8(at, cuda(scale), wp, cuda(s_w), mean=mean_t, w_rowsum=w1_t, bias=bias_t)
    torch.cuda.synchronize()
    assert oq.device_status()[0] == 0
    ref = oracle.epilogue(oracle.gemm_int(a, w), scale.astype(np.float64),
                          s_w.astype(np.float64), mean.astype(np.float64) if with_mean else None,
                          w1.astype(np.float64) if with_mean else None,
                          synth.bf16_to_f64(bias_bits) if with_bias else None)
    got = y.float().cpu().numpy().astype(np.float64)
    assert rel_fro(got, ref) < 3e-3
    # token rows are independent: the first row alone gives the same bits
    y1 = oq.gemm_w4a8(at[:1], cuda(scale[:1]), wp, cuda(s_w),
                      mean=mean_t[:1] if with_mean else None, w_rowsum=w1_t, bias=bias_t)
    torch.cuda.synchronize()
    assert torch.equal(y1[0], y[0])
