"""GPU parity of the asymmetric grouped INT4 weights (CentriQ Eq. 2, §4.3, App. B.2).

- Weight preparation: sigma, z (fp16) and the codes Q - 8 against the float64 oracle run on the
  bf16 weights: sigma and z identical except in groups whose float64 value lies within 1e-5
  relative of an fp16 rounding boundary, codes identical except where w / sigma + z lies within
  1e-5 relative of a rounding boundary k + 1/2 (the exempted counts are printed).
- GEMM: the fp32 accumulators against (a) the fp64 sum over the exact fp16 operand the
  converters build, sigma (Q - 8) + fp16(sigma (8 - z)) rounded once to fp16, and (b) the
  oracle's exact dequantized weights sigma (Q - z), within the bound derived from two fp16
  roundings per weight (u = 2^-11):
      |acc - acc_exact| <= u sum_k |a_k| (|w_k| + 1.01 |m_g|) + K 2^-24 sum_k |a_k w_k|,
  the last term a worst case for fp32 accumulation over K products.
- The layer: bf16 outputs within 8e-3 relative (Frobenius) of the float64 oracle, on a
  reduced token count and on sampled rows of the full-size workload.
"""
import numpy as np
import pytest

import oracle
import synth
from oracle import weights_g64 as G
from parity import (OUT_TOL, fp16_boundary_mask, grid_boundary_mask, pack_w4_gemm, rel_fro,
                    to_torch_bf16, unpack_w4_gemm)

pytestmark = pytest.mark.gpu

U16 = 2.0 ** -11


def _k_order(d):
    """Stored K order of the grouped weights: position p holds column pi(p), pi swapping bits 0
    and 1 of the index (an involution), so natural = stored[:, pi] and stored = natural[:, pi]."""
    k = np.arange(d)
    return (k & ~3) | ((k & 1) << 1) | ((k >> 1) & 1)


def _split_sz(wsz):
    """int32 [G, N] words -> (sigma, z) float64 [N, G]."""
    w = np.ascontiguousarray(wsz).view(np.uint32)
    s = (w & 0xFFFF).astype(np.uint16).view(np.float16).astype(np.float64)
    z = (w >> 16).astype(np.uint16).view(np.float16).astype(np.float64)
    return s.T.copy(), z.T.copy()


def _pack_sz(s, z):
    """(sigma, z) [N, G] -> int32 [G, N] words (fp16 bits)."""
    sb = np.asarray(s, np.float16).view(np.uint16).astype(np.uint32)
    zb = np.asarray(z, np.float16).view(np.uint16).astype(np.uint32)
    return np.ascontiguousarray((sb | (zb << 16)).T).view(np.int32)


@pytest.mark.parametrize("n_out,d,h,rounds", [(256, 256, 64, 1), (208, 3072, 1024, 1),
                                              (1920, 1920, 128, 2), (48, 4096, 512, 1),
                                              (64, 512, 1, 1)])
def test_prepare_weights_g64_matches_fp64_oracle(n_out, d, h, rounds):
    import torch
    import w4a8_ptq_linear_b200 as oq
    wb = synth.make_w(n_out, d, seed=7)
    wb[3, :] = synth.f64_to_bf16(np.full(d, 0.125))   # a constant row
    if h == 1:
        # a rotated group that is constant and far from zero (its shift would overflow fp16
        # without the |min| / 2^15 floor on sigma): with h = 1 a round only permutes and signs,
        # so the row that rotates to it is exact in bf16
        pl = oracle.rpbh_plan(d, 1, 1, 0)
        tr = oracle.rotate(synth.bf16_to_f64(wb[5:6]), pl, 1)
        tr[0, :64] = 6.5
        wb[5] = synth.f64_to_bf16(oracle.unrotate(tr, pl, 1)[0])
    wt = to_torch_bf16(wb)
    plan = oq.Plan(d, h, rounds)
    wp, wsz, ws, w1 = oq.prepare_weights_g64(plan, wt)
    torch.cuda.synchronize()
    st, code = oq.device_status()
    assert st == 0, hex(code)
    w = synth.bf16_to_f64(wb)
    # the float64 definition on the bf16 weights (no GPU value enters the reference)
    w_r = oracle.rotate(w, oracle.rpbh_plan(d, h, rounds, 0), h)
    q, s, z = G.asym_group_quantize(w_r, store=np.float16)
    gs, gz = _split_sz(wsz.cpu().numpy())
    # float64 values before the fp16 rounding, for the boundary exemptions
    wg = w_r.reshape(n_out, d // 64, 64)
    lo, hi = wg.min(axis=2), wg.max(axis=2)
    s64 = np.maximum(np.maximum((hi - lo) / 15, G.SIGMA_MIN_F16), np.abs(lo) / G.SHIFT_MAX)
    ex_s = fp16_boundary_mask(s64)
    ex_z = fp16_boundary_mask(-lo / s, floor=1.0)
    ex_g = ex_s | ex_z                                 # groups whose grid may differ
    assert np.array_equal(gs[~ex_s], s[~ex_s])
    assert np.array_equal(gz[~ex_g], z[~ex_g])
    assert np.all(np.isfinite(gz))
    if h == 1:
        assert np.all(wg[5, 0] == 6.5) and np.abs(gz[5, 0]) < 65504
    codes = unpack_w4_gemm(wp.cpu().numpy())[:, _k_order(d)] + 8
    v = wg / s[..., None] + z[..., None]
    ex_c = grid_boundary_mask(v, 0, 15).reshape(n_out, d) | np.repeat(ex_g, 64, axis=1)
    bad = int(np.sum((codes != q) & ~ex_c))
    print(f"g64 prep n_out={n_out} d={d}: {int(ex_s.sum())} sigma and {int(ex_z.sum())} z "
          f"exemptions of {ex_s.size} groups, {int(ex_c.sum())} exempt codes of {q.size}")
    assert bad == 0, f"{bad} codes differ outside the boundary exemption"
    assert np.all(ws.cpu().numpy() == 1.0)
    assert np.all(np.abs(w1.cpu().numpy() - w.sum(axis=1)) <= 1e-5 * np.abs(w).sum(axis=1))
    # every weight is within half a grid step of its reconstruction (the fp16 shift moves the
    # grid by at most half an ulp of z)
    err = np.abs(G.dequantize(codes, gs, gz) - w_r).reshape(n_out, d // 64, 64)
    step = gs * (0.5 + 2.0 ** -11 * np.maximum(1.0, np.abs(gz)) + 1e-4)
    assert np.all(err <= step[..., None])
    plan.close()


def _operands(rng, T, K, N):
    a = rng.integers(-7, 8, (T, K))
    a[0, :] = 7
    q = rng.integers(0, 16, (N, K))
    s = rng.uniform(2e-3, 4e-2, (N, K // 64)).astype(np.float16).astype(np.float64)
    z = rng.uniform(-2.0, 17.0, (N, K // 64)).astype(np.float16).astype(np.float64)
    s[1, :] = 2.0 ** -14                                        # the sigma floor
    return a, q, s, z


def _kernel_operand(q, s, z):
    """The fp16 weight the converters build: fp16(sigma (Q - 8) + fp16(f32(sigma) * f32(8 - z)))."""
    m = (s.astype(np.float32) * (np.float32(8) - z.astype(np.float32))).astype(np.float16)
    m = np.repeat(m.astype(np.float64), 64, axis=1)
    sr = np.repeat(s, 64, axis=1)
    return (sr * (q - 8) + m).astype(np.float16).astype(np.float64)


@pytest.mark.parametrize("T,K,N", [(64, 256, 256), (200, 384, 272), (300, 3072, 3072),
                                   (7, 128, 16), (2560, 1536, 2560)])
def test_g64_accumulators_and_epilogue(T, K, N):
    import torch
    import w4a8_ptq_linear_b200 as oq
    rng = np.random.default_rng(3 * T + K + N)
    a, q, s, z = _operands(rng, T, K, N)
    cu = lambda v: torch.from_numpy(np.ascontiguousarray(v)).cuda()
    ap, wsz = cu(oracle.pack_nibbles(a)), cu(_pack_sz(s, z))
    wp = cu(pack_w4_gemm((q - 8)[:, _k_order(K)]))
    ones = torch.ones(max(T, N), dtype=torch.float32, device="cuda")
    acc = oq.gemm_w4a4_g64("int4_absmax", ap, ones[:T], wp, wsz, ones[:N], out_kind=oq.OUT_ACC)
    alpha = rng.uniform(0.5, 2.0, T)
    mean = rng.standard_normal(T)
    w1 = rng.standard_normal(N)
    bias = synth.f64_to_bf16(rng.standard_normal(N) * 0.1)
    y = oq.gemm_w4a4_g64("int4_absmax", ap, cu(alpha.astype(np.float32)), wp, wsz, ones[:N],
                         mean=cu(mean.astype(np.float32)), w_rowsum=cu(w1.astype(np.float32)),
                         bias=to_torch_bf16(bias))
    torch.cuda.synchronize()
    st, code = oq.device_status()
    assert st == 0, hex(code)
    got = acc.cpu().numpy().astype(np.float64)
    af = a.astype(np.float64)
    wk = _kernel_operand(q, s, z)
    ref_k = af @ wk.T                          # (a) the operand the kernel builds
    mag = np.abs(af) @ np.abs(wk).T
    acc_tol = K * 2.0 ** -24 * mag
    assert np.all(np.abs(got - ref_k) <= acc_tol + 1e-30)
    wx = G.dequantize(q, s, z)                 # (b) the oracle's exact weights
    ref_x = af @ wx.T
    mg = np.repeat(np.abs(s * (z - 8)), 64, axis=1)
    bound = U16 * (np.abs(af) @ (np.abs(wx) + 1.01 * mg).T) + acc_tol
    assert np.all(np.abs(got - ref_x) <= bound)
    # the App. B.2 form of the same product
    assert np.allclose(G.corrected_product(a, q, s, z), ref_x, rtol=0,
                       atol=1e-9 * np.abs(ref_x).max())
    ref_y = oracle.epilogue(ref_x, alpha.astype(np.float32), np.ones(N),
                            mean.astype(np.float32), w1.astype(np.float32),
                            synth.bf16_to_f64(bias))
    assert rel_fro(y.float().cpu().numpy(), ref_y) <= 3e-3


def _gpu_layer(wl, xb, wb):
    import torch
    import w4a8_ptq_linear_b200 as oq
    plan = oq.Plan(wl.d, wl.h, wl.rounds, seed=wl.seed, center=wl.center, act=wl.act)
    wp, wsz, ws, w1 = oq.prepare_weights_g64(plan, to_torch_bf16(wb))
    y = oq.linear_g64(plan, to_torch_bf16(xb), wp, wsz, ws, w1)
    torch.cuda.synchronize()
    st, code = oq.device_status()
    assert st == 0, hex(code)
    out = y.float().cpu().numpy().astype(np.float64)
    plan.close()
    return out


def _oracle_rows(wl, xb_rows, wb):
    plan = oracle.rpbh_plan(wl.d, wl.h, wl.rounds, wl.seed)
    y, _, _ = G.linear_forward_g64(synth.bf16_to_f64(xb_rows), synth.bf16_to_f64(wb), plan,
                                   wl.h, wl.act, wl.center)
    return y


@pytest.mark.parametrize("T", [130, 1])
def test_g64_layer_matches_oracle(T):
    wl, xb, wb = synth.make_inputs("mlp_up_g64", T=T)
    y = _gpu_layer(wl, xb, wb)
    assert rel_fro(y, _oracle_rows(wl, xb, wb)) <= OUT_TOL


def test_g64_full_size_layer_on_sampled_rows():
    wl, xb, wb = synth.make_inputs("mlp_up_g64")
    y = _gpu_layer(wl, xb, wb)
    rows = np.sort(np.random.default_rng(42).choice(wl.T, 48, replace=False))
    rows = np.unique(np.concatenate([rows, [0, wl.T - 1]]))
    assert rel_fro(y[rows], _oracle_rows(wl, xb[rows], wb)) <= OUT_TOL
    assert np.all(np.isfinite(y))


def test_g64_beats_per_channel_weights():
    # groups of 64 follow the local range: the layer error against the unquantized layer is
    # below that of the per-channel symmetric weights on the same activations
    wl, xb, wb = synth.make_inputs("mlp_up_g64", T=96)
    y_g = _gpu_layer(wl, xb, wb)
    plan = oracle.rpbh_plan(wl.d, wl.h, wl.rounds, wl.seed)
    y_ref = oracle.linear_unquantized(synth.bf16_to_f64(xb), synth.bf16_to_f64(wb), plan, wl.h,
                                      wl.center)
    y_c, _, _ = oracle.linear_forward(synth.bf16_to_f64(xb), synth.bf16_to_f64(wb), plan, wl.h,
                                      wl.act, wl.center)
    assert rel_fro(y_g, y_ref) < rel_fro(y_c, y_ref)
