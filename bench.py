#!/usr/bin/env python
"""Benchmark of the rotated, quantized linear layer on B200.

One step = one pass of the whole hot path over one batch of tokens: the fused
center + RPBH + quantize kernel followed by the tcgen05 low-bit GEMM with its dequant
epilogue (weights are prepared once, offline, before timing). Default workload: the
DiT-width W4A8 layer, T = 4096 tokens, d_in = d_out = 3072, block h = 1024, one round,
absmax INT8 activations, INT4 per-channel weights.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME]
  python bench.py --sweep      # rotate+quantize bandwidth at every sweep point (one GPU)

Multi-GPU (launched by torchrun, one process per GPU): tokens are independent, so every rank
runs its own batch with no collective on the data path (weak scaling); the only collectives
are the barriers around the timed region and the max-over-ranks of the time.

Timing: CUDA events on the launching stream over exactly K steps, a barrier and a
synchronize on both sides. The steps replay CUDA graphs of the library's launches (one graph
of four steps, plus single steps for a remainder), so that no host-side launch gap falls
between kernels. Inputs rotate over 4 independent sets (about 270 MB, more than the 126 MB
L2), so no step reads data a previous step left in L2. Per-kernel durations come from graphs
of each kernel alone over the same sets. The GEMM's roofline peak is the library's tcgen05
peak loop for the GEMM's MMA kind, measured in the same run. nvidia-smi samples the SM clock
and throttle reasons during the timed region.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "rotate+quantize GB/s (% of HBM peak); W4A8/W4A4 linear TOPS (% tensor peak)"
RING = 4            # independent input sets at least; more when a set is small (see ring_size)
L2_BYTES = 126 << 20   # B200 L2
# nominal dense int8 / bf16 tensor throughput ratio on B200 (4.5 / 2.25 PFLOP/s), for the
# peak the measured bf16 GEMM figure implies (reported beside the measured tcgen05 peak)
INT8_PER_BF16 = 2.0
# activation kinds the single-launch layer takes
FUSED_ACTS = ("int8_absmax", "int4_absmax", "int4_percentile")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch from an ncu capture, valid only for the kernel source it was taken
# on (sha256 of the kernel's source files at capture time); null once they have changed.
NCU_TRAFFIC = {
    # ncu --set full of k_gemm_a8s (profiles/k_gemm_dit_w4a8.md): dram read 17.378 MB + write 0.028 MB
    ("dit_w4a8", "k_gemm"): {"sha": "1cd5718ddffa4e06462ea9fe112d66be691be407e62728f26e7033b23e0691b6", "bytes": 17406464},
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum of k_rotate_quant_pair<10, 1, 0>
    # (profiles/k_rotate_quant_dit_w4a8.md): dram read 25.229 MB + write 0
    ("dit_w4a8", "k_rotate_quant"): {"sha": "4b015d18928769dad475d94b8ec7157548036b65a5e9d65eb4b1d2098617a6c8", "bytes": 25229312},
    # the same metrics of k_linear_fused<10, 1, 1, 0> at T = 256 (profiles/k_linear_fused_t256.md):
    # dram read 3.294 MB + write 0
    ("dit_w4a8@T256", "k_linear_fused"): {"sha": "8d5c5d5381a3e22bfb7dd801e3c23b1639653c392cdaf29e5f574263b7ab32a9", "bytes": 3294464},
    # the same metrics of the split-K GEMM k_linear_fused<0, 1, 0, 0> at T = 256
    # (profiles/k_gemm_splitk_t256.md): dram read 5.558 MB + write 0
    ("dit_w4a8@T256", "k_gemm"): {"sha": "8d5c5d5381a3e22bfb7dd801e3c23b1639653c392cdaf29e5f574263b7ab32a9", "bytes": 5558272, "sources": "k_linear_fused"},
}


def parse():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="dit_w4a8",
                    choices=["tiny", "dit_w4a8", "dit_a4", "dit_lm8", "narrow_lm", "narrow_lm_w",
                             "mlp_up", "mlp_up_pct", "mlp_up_a2", "mlp_up_g64"])
    ap.add_argument("--fused", action="store_true",
                    help="time the single-launch layer (oq_linear_fused; INT8 absmax, INT4 "
                         "absmax or percentile activations, T <= 256)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the token count (small cases for profiler captures)")
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU time budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="time rotate+quantize alone at every point of the bandwidth sweep "
                         "(T x d x h x rounds x output), one JSON line per point")
    ap.add_argument("--sweep-iters", type=int, default=10)
    ap.add_argument("--peaks", action="store_true",
                    help="measure the dense tensor-core peaks on this GPU: the library's "
                         "tcgen05 peak loop (kind::i8, kind::f16) and cuBLAS int8 / bf16 "
                         "GEMMs at 8192^3, with the SM clock sampled")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---- multi-rank host logic (one process per GPU; each rank runs the whole path on its own
# shard of independent token batches, so there is no collective on the data path) ----------
def input_seed(base_seed, rank, r):
    """Seed of input set r on `rank`: every rank draws different tokens of the same shape."""
    return base_seed + 1000 * rank + r


def max_over_ranks(x, world, dist=None, device=None):
    """The largest value of the scalar x over all ranks (one all-reduce when world > 1)."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms):
    """Units per second of the whole job: every rank processed units_per_rank in at most ms."""
    return units_per_rank * world / (ms * 1e-3)


def sha_of(*paths):
    """sha256 of the kernel sources a traffic figure was taken with (concatenated)."""
    h = hashlib.sha256()
    for path in paths:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def csrc(name):
    return os.path.join(ROOT, "w4a8_ptq_linear_b200", "csrc", name)


# the sources each kernel's DRAM traffic depends on
KERNEL_SOURCES = {
    "k_gemm": ("k_gemm.cu", "ptx.cuh"),
    "k_rotate_quant": ("rq_device.cuh", "k_rotate_quant.cu", "ptx.cuh"),
    "k_linear_fused": ("k_linear_fused.cu", "rq_device.cuh", "ptx.cuh"),
}


def ncu_traffic(workload, kernel):
    """DRAM bytes per launch from the committed ncu capture, or None once the kernel's sources
    have changed since it was taken."""
    tr = NCU_TRAFFIC.get((workload, kernel))
    if not tr:
        return None
    files = KERNEL_SOURCES[tr.get("sources", kernel)]
    return tr["bytes"] if tr["sha"] == sha_of(*[csrc(f) for f in files]) else None


# ---- clocks ---------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid, enabled=True):
        self.uuid = uuid
        self.proc = None
        self.enabled = enabled
        self.path = None

    def __enter__(self):
        if not self.enabled:
            return self
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["not sampled"]}
        rows = []
        with open(self.path) as f:
            for r in csv.reader(f):
                r = [c.strip() for c in r]
                if len(r) < 9:
                    continue
                if self.uuid and r[0] != self.uuid:
                    continue
                rows.append(r)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows
                                    if r[3].replace(".", "").isdigit()), default=None)}


# ---- CPU oracle legs ---------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_setup(wl, x_bits, w_bits):
    import numpy as np
    import oracle
    import synth
    plan = oracle.rpbh_plan(wl.d, wl.h, wl.rounds, wl.seed)
    c, t = (oracle.lloyd_max_sphere(wl.d) if wl.act == "int4_lloydmax_width"
            else oracle.lloyd_max_gaussian_8bit() if wl.act == "int8_lloydmax"
            else oracle.lloyd_max_gaussian())
    if wl.weights == "int4_g64":
        from oracle import weights_g64
        q, sg, z, w1 = weights_g64.prepare_weights_g64(synth.bf16_to_f64(w_bits), plan, wl.h)
        return plan, c, t, weights_g64.dequantize(q, sg, z), np.ones(wl.n_out), w1
    w_codes, s_w, w1 = oracle.prepare_weights(synth.bf16_to_f64(w_bits), plan, wl.h)
    return plan, c, t, w_codes, s_w, w1


def oracle_pass(wl, setup, x_rows_f64):
    import oracle
    plan, c, t, w_codes, s_w, w1 = setup
    qa = oracle.quantize_activations(x_rows_f64, plan, wl.h, wl.act, wl.center, t)
    if "lloydmax" in wl.act:
        acc = oracle.gemm_lloyd_max(qa["codes"], c, w_codes)
    elif wl.weights == "int4_g64":   # w_codes holds the dequantized grouped weights
        acc = qa["codes"].astype(float) @ w_codes.T
    else:
        acc = oracle.gemm_int(qa["codes"], w_codes)
    return oracle.epilogue(acc, qa["scale"], s_w, qa["mean"] if wl.center else None,
                           w1 if wl.center else None)


def cpu_baseline(wl, x_bits, w_bits, seconds):
    import synth
    setup = oracle_setup(wl, x_bits, w_bits)
    n = min(1024, wl.T)
    xs = synth.bf16_to_f64(x_bits[:n])
    done, t0 = 0, time.perf_counter()
    while True:
        oracle_pass(wl, setup, xs)
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds or done >= 64:
            break
    ops = 2.0 * n * wl.d * wl.n_out * done
    return {"value": ops / el / 1e12, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{done} pass(es) of the oracle over {n} of the {wl.T} tokens "
                      f"(float64 NumPy, weights prepared beforehand), {el:.1f} s"}


def run_reference(args, wl, rank):
    """--impl reference: the CPU oracle, as it stands, timed on the host cores."""
    if rank != 0:
        return None
    import numpy as np
    import synth
    T = args.tokens or wl.T
    wl_, x_bits, w_bits = synth.make_inputs(wl.name, T=min(T, 1024))
    setup = oracle_setup(wl, x_bits, w_bits)
    xs = synth.bf16_to_f64(x_bits)
    # size each step so that warm-up + K steps take about two minutes in total
    t0 = time.perf_counter()
    oracle_pass(wl, setup, xs[:8])
    per_tok = (time.perf_counter() - t0) / 8
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(len(xs), budget / max(per_tok, 1e-6))))
    for i in range(args.warmup):
        oracle_pass(wl, setup, xs[:n])
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_pass(wl, setup, xs[(i * n) % (len(xs) - n + 1):][:n])
    el = time.perf_counter() - t0
    ops = 2.0 * n * wl.d * wl.n_out * args.steps
    v = ops / el / 1e12
    sample = f"{n} tokens per step of the {T}-token workload (float64 NumPy oracle)"
    return {"metric": METRIC, "value": v, "unit": "TOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": config_of(wl, T, args.gpus, fused=args.fused),
            "cpu_baseline": {"value": v, "unit": "TOPS", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "TOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def set_bytes(wl, T):
    """Device bytes of one input set: activations, prepared weights, codes, scales, output."""
    code = (T * wl.d if wl.act.startswith("int8")
            else T * wl.d // 4 if wl.act.startswith("int2") else T * wl.d // 2)
    return T * wl.d * 2 + wl.n_out * wl.d // 2 + 12 * wl.n_out + code + 8 * T + T * wl.n_out * 2


def ring_size(wl, T, l2_bytes):
    """Input sets the timed steps rotate over: at least RING, and together at least twice the
    L2, so that every step reads its weights and activations from HBM as a layer of a real
    model would (capped at 256 sets)."""
    return int(min(256, max(RING, -(-2 * l2_bytes // set_bytes(wl, T)))))


def config_of(wl, T, n, ring=None, l2_bytes=L2_BYTES, fused=False):
    ring = ring_size(wl, T, l2_bytes) if ring is None else ring
    c = {"workload": wl.name, "T": T, "d_in": wl.d, "d_out": wl.n_out, "h": wl.h,
         "rounds": wl.rounds, "act": wl.act, "center": wl.center,
         "weights": "int4" if wl.weights == "int4_channel" else wl.weights,
         "l2": (f"inputs rotate over {ring} sets, {ring * set_bytes(wl, T) / 1e6:.0f} MB "
                f"together, larger than the {l2_bytes / 1e6:.0f} MB L2"),
         "parallelism": "replicas" if n == 1 else f"dp{n} (tokens split, no collective)"}
    if fused:
        c["path"] = "single launch (oq_linear_fused)"
    return c


# ---- GPU leg ---------------------------------------------------------------------------------
def run_sweep(args):
    """Rotate+quantize alone at every sweep point. Inputs are drawn on the device (N(0,1) plus
    a per-token mean of variance 3, bf16); the L2 is flushed by writing a 256 MB buffer before
    every timed launch, and each launch is timed by CUDA events on its stream."""
    import torch
    import synth
    import w4a8_ptq_linear_b200 as oq
    peaks, peak_kind = load_peaks()
    hbm = peaks["hbm_gbs"]
    dev = torch.device("cuda", 0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    gen = torch.Generator(device=dev)
    for (T, d, h, rounds, act) in synth.sweep_points():
        plan = oq.Plan(d, h, rounds, seed=0, center=False, act=act)
        gen.manual_seed(1000003 * T + d)
        x = (torch.randn((T, d), generator=gen, device=dev) +
             3.0 ** 0.5 * torch.randn((T, 1), generator=gen, device=dev)).to(torch.bfloat16)
        codes, scale, _, _ = oq.rotate_quantize(plan, x)
        times = []
        for i in range(args.warmup + args.sweep_iters):
            flush.fill_(i & 0xFF)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            oq.rotate_quantize(plan, x, codes=codes, scale=scale)
            e1.record()
            torch.cuda.synchronize()
            if i >= args.warmup:
                times.append(e0.elapsed_time(e1))
        st, code = oq.device_status()
        if st != 0:
            raise RuntimeError(f"device status {st} code {code:#x} at sweep point {T, d, h}")
        ms = sum(times) / len(times)
        nbytes = T * d * 2 + (T * d if act == "int8_absmax" else T * d // 2) + 4 * T
        gbs = nbytes / (ms * 1e-3) / 1e9
        print(json.dumps({"sweep": {"T": T, "d": d, "h": h, "rounds": rounds, "act": act},
                          "us": ms * 1e3, "gbs": gbs, "frac_hbm": gbs / hbm,
                          "peak": f"{peak_kind} copy bandwidth {hbm} GB/s",
                          "l2": "flushed before every launch", "iters": len(times)}),
              flush=True)
        del x, codes, scale
        plan.close()
    return 0


def measured_mma_peak(oq, kind, stream, iters=1 << 13, reps=3):
    """(TOPS or TFLOP/s, ms) of the library's tcgen05 peak loop for `kind` ("i8" or "f16"),
    best of `reps` launches timed with CUDA events on `stream`."""
    import torch
    k_per = 32 if kind == "i8" else 16
    pairs = oq.mma_peak_loop(kind, iters, stream=stream)
    best = None
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        oq.mma_peak_loop(kind, iters, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        best = ms if best is None else min(best, ms)
    st, code = oq.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} code {code:#x} in the peak loop")
    ops = pairs * iters * 4 * 2.0 * 256 * 256 * k_per
    return ops / (best * 1e-3) / 1e12, best


def run_peaks(args):
    """Dense tensor-core peaks of this GPU, each timed with CUDA events on its stream after
    warm-up, best of `reps`:
      - tcgen05 loop: oq_mma_peak_loop, the GEMMs' own instruction (cta_group::2, M = N = 256)
        issued back to back on shared-memory operands, one CTA pair per two SMs;
      - cuBLAS: torch._int_mm (int8 x int8 -> int32) and torch.matmul (bf16) at 8192^3.
    One JSON line per measurement, with the SM clock and throttle reasons sampled during it."""
    import torch
    import w4a8_ptq_linear_b200 as oq
    dev = torch.device("cuda", 0)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    reps = 10

    def timed(fn, n_inner):
        fn()
        torch.cuda.synchronize()
        best = None
        with ClockSampler(uuid, enabled=not args.no_clocks) as clk:
            for _ in range(reps):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(n_inner):
                    fn()
                e1.record()
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1) / n_inner
                best = ms if best is None else min(best, ms)
        return best, clk.summary()

    out = []
    group_us = {}
    for kind, k_per in (("i8", 32), ("f16", 16), ("i8_serial", 32)):
        iters = 1 << 14
        pairs = oq.mma_peak_loop(kind, iters)
        ms, clocks = timed(lambda: oq.mma_peak_loop(kind, iters), 4)
        ops = pairs * iters * 4 * 2.0 * 256 * 256 * k_per
        st, code = oq.device_status()
        if st != 0:
            raise RuntimeError(f"device status {st} code {code:#x} in the peak loop")
        group_us[kind] = ms * 1e3 / iters
        line = {"peak": f"tcgen05 kind::{kind} loop", "value": ops / (ms * 1e-3) / 1e12,
                "unit": "TOPS" if kind != "f16" else "TFLOP/s", "ms": ms, "pairs": pairs,
                "us_per_group_of_four": group_us[kind], "clocks": clocks}
        if kind == "i8_serial":
            # each group waited for before the next: the extra time per group is the latency
            # from the end of the MMAs to the completion the issuing thread sees
            line["completion_latency_us"] = group_us["i8_serial"] - group_us["i8"]
        out.append(line)
    n = 8192
    a8 = torch.randint(-128, 128, (n, n), dtype=torch.int8, device=dev)
    b8 = torch.randint(-128, 128, (n, n), dtype=torch.int8, device=dev)
    ms, clocks = timed(lambda: torch._int_mm(a8, b8), 1)
    out.append({"peak": "cuBLAS int8 GEMM (torch._int_mm) 8192^3",
                "value": 2.0 * n ** 3 / (ms * 1e-3) / 1e12, "unit": "TOPS", "ms": ms,
                "clocks": clocks})
    del a8, b8
    ab = torch.randn((n, n), dtype=torch.bfloat16, device=dev)
    bb = torch.randn((n, n), dtype=torch.bfloat16, device=dev)
    ms, clocks = timed(lambda: torch.matmul(ab, bb), 1)
    out.append({"peak": "cuBLAS bf16 GEMM (torch.matmul) 8192^3",
                "value": 2.0 * n ** 3 / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms": ms,
                "clocks": clocks})
    for o in out:
        print(json.dumps(o), flush=True)
    return 0


def main():
    args = parse()
    if args.sweep:
        return run_sweep(args)
    if args.peaks:
        return run_peaks(args)
    import synth
    wl = synth.WORKLOADS[args.workload]
    T = args.tokens or wl.T
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, wl, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    import numpy as np
    import torch
    import torch.distributed as dist
    import w4a8_ptq_linear_b200 as oq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    _, _, w_bits = synth.make_inputs(wl.name, T=1)
    g64 = wl.weights == "int4_g64"
    plan = oq.Plan(wl.d, wl.h, wl.rounds, seed=wl.seed, center=wl.center, act=wl.act)
    to_dev = lambda b: torch.from_numpy(np.ascontiguousarray(b)).view(torch.bfloat16).to(dev)

    # independent sets: activations, prepared weights, codes, scales, outputs
    ring = ring_size(wl, T, L2_BYTES)
    fused = args.fused
    if fused and (wl.act not in FUSED_ACTS or g64 or T > 256):
        raise SystemExit("--fused takes INT8 absmax or INT4 absmax / percentile workloads with "
                         "per-channel weights, T <= 256")
    sets = []
    x_host_bits = None
    for r in range(ring):
        xb = synth.make_x(T, wl.d, mean_var=wl.mean_var, heavy_frac=wl.heavy_frac,
                          outliers=wl.outliers, outlier_gain=wl.outlier_gain,
                          seed=input_seed(wl.seed, rank, r))
        if r == 0:
            x_host_bits = xb
        w = to_dev(w_bits)
        wsz = None
        if g64:
            wp, wsz, ws, w1 = oq.prepare_weights_g64(plan, w)
        else:
            wp, ws, w1 = oq.prepare_weights(plan, w)
        del w
        s = {"x": to_dev(xb), "wp": wp, "ws": ws, "w1": w1, "wsz": wsz,
             "codes": torch.empty((T, plan.code_row_bytes),
                                  dtype=torch.int8 if wl.act == "int8_absmax" else torch.uint8,
                                  device=dev),
             "scale": torch.empty(T, dtype=torch.float32, device=dev),
             "mean": torch.empty(T, dtype=torch.float32, device=dev) if wl.center else None,
             "y": torch.empty((T, wl.n_out), dtype=torch.bfloat16, device=dev)}
        if fused:
            s["wsb"] = torch.empty(max(plan.workspace_bytes(T), 256), dtype=torch.uint8,
                                   device=dev)
        sets.append(s)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def step(s, st):
        if fused:   # the whole layer in one launch
            oq.linear_fused(plan, s["x"], s["wp"], s["ws"], s["w1"] if wl.center else None,
                            workspace=s["wsb"], out=s["y"], stream=st)
            return
        oq.rotate_quantize(plan, s["x"], codes=s["codes"], scale=s["scale"], mean=s["mean"],
                           stream=st)

    def gemm(s, st):
        if fused:
            return
        if g64:
            oq.gemm_w4a4_g64(wl.act, s["codes"], s["scale"], s["wp"], s["wsz"], s["ws"],
                             mean=s["mean"], w_rowsum=s["w1"] if wl.center else None, out=s["y"],
                             stream=st)
        elif wl.act == "int8_absmax":
            oq.gemm_w4a8(s["codes"], s["scale"], s["wp"], s["ws"], mean=s["mean"],
                         w_rowsum=s["w1"] if wl.center else None, out=s["y"], stream=st)
        elif wl.act == "int2_percentile":
            oq.gemm_w4a2(s["codes"], s["scale"], s["wp"], s["ws"], mean=s["mean"],
                         w_rowsum=s["w1"] if wl.center else None, out=s["y"], stream=st)
        elif wl.act == "int8_lloydmax":
            oq.gemm_w4a8_lloydmax(plan, s["codes"], s["scale"], s["wp"], s["ws"], mean=s["mean"],
                                  w_rowsum=s["w1"] if wl.center else None, out=s["y"],
                                  stream=st)
        else:
            oq.gemm_w4a4(plan, wl.act, s["codes"], s["scale"], s["wp"], s["ws"],
                         mean=s["mean"], w_rowsum=s["w1"] if wl.center else None, out=s["y"],
                         stream=st)

    for i in range(max(3, args.warmup)):
        s = sets[i % ring]
        step(s, stream)
        gemm(s, stream)
    torch.cuda.synchronize()
    st, code = oq.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} code {code:#x} after warm-up")

    # The timed steps replay CUDA graphs of the library's launches, so that no host-side launch
    # gap falls between the kernels: g_ring holds the ring's steps in order, g_one[r] one step.
    cap_stream = torch.cuda.Stream(device=dev)

    def capture(calls):
        g = torch.cuda.CUDAGraph()
        cap_stream.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap_stream):
            cs = torch.cuda.current_stream()
            for fn, s in calls:
                fn(s, cs)
        stream.wait_stream(cap_stream)
        return g

    g_ring = capture([(f, s) for s in sets for f in (step, gemm)])
    g_one = [capture([(step, s), (gemm, s)]) for s in sets]
    g_rq = capture([(step, s) for s in sets])        # the two kernels alone, for their
    g_gm = None if fused else capture([(gemm, s) for s in sets])   # average duration per launch
    for _ in range(2):
        g_ring.replay()
    torch.cuda.synchronize()

    K = args.steps
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(uuid, enabled=not args.no_clocks) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for _ in range(K // ring):
            g_ring.replay()
        for r in range(K % ring):
            g_one[r].replay()
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    elapsed_ms = t_start.elapsed_time(t_end)

    def per_launch(g):
        reps = max(1, -(-K // ring))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / (reps * ring)

    rq_ms = per_launch(g_rq)
    gm_ms = per_launch(g_gm) if g_gm is not None else 0.0
    st, code = oq.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} code {code:#x} after timing")

    elapsed_ms = max_over_ranks(elapsed_ms, world, dist, dev)
    clocks = clk.summary()

    # ---- end to end through the public API with host buffers ------------------------------
    # Every step copies its input from pinned host memory, runs oq_linear and copies the
    # result back. Three streams (host->device, the layer, device->host) and two device buffer
    # sets let step i's input copy overlap step i-1's layer and step i-2's output copy, as a
    # serving loop would; events order each buffer's reuse.
    NB = 2
    x_pin = torch.from_numpy(np.ascontiguousarray(x_host_bits)).view(torch.bfloat16).pin_memory()
    y_pins = [torch.empty((T, wl.n_out), dtype=torch.bfloat16).pin_memory() for _ in range(NB)]
    s0 = sets[0]
    ws_bytes = plan.workspace_bytes(T)
    workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    x_devs = [torch.empty_like(s0["x"]) for _ in range(NB)]
    y_devs = [torch.empty_like(s0["y"]) for _ in range(NB)]
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(NB)]     # input k copied to the device
    ev_done = [torch.cuda.Event() for _ in range(NB)]   # layer on buffer set k finished
    ev_out = [torch.cuda.Event() for _ in range(NB)]    # output k copied to the host

    def e2e_step(i):
        k = i % NB
        s_in.wait_event(ev_done[k])          # step i - NB no longer reads x_devs[k]
        with torch.cuda.stream(s_in):
            x_devs[k].copy_(x_pin, non_blocking=True)
        ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        stream.wait_event(ev_out[k])         # step i - NB's output has left y_devs[k]
        if g64:
            oq.linear_g64(plan, x_devs[k], s0["wp"], s0["wsz"], s0["ws"],
                          s0["w1"] if wl.center else None, workspace=workspace, out=y_devs[k],
                          stream=stream)
        else:
            layer = oq.linear_fused if fused else oq.linear
            layer(plan, x_devs[k], s0["wp"], s0["ws"], s0["w1"] if wl.center else None,
                  workspace=workspace, out=y_devs[k], stream=stream)
        ev_done[k].record(stream)
        s_out.wait_event(ev_done[k])
        with torch.cuda.stream(s_out):
            y_pins[k].copy_(y_devs[k], non_blocking=True)
        ev_out[k].record(s_out)

    def drain():
        for k in range(NB):
            stream.wait_event(ev_out[k])

    for i in range(3):
        e2e_step(i)
    drain()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for i in range(args.e2e_steps):
        e2e_step(i)
    drain()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, dist, dev)
    barrier()

    # ---- numbers ------------------------------------------------------------------------------
    ops = 2.0 * T * wl.d * wl.n_out
    ms_per_step = elapsed_ms / K
    value = whole_job_rate(ops, world, ms_per_step) / 1e12
    code_bytes = (T * wl.d if wl.act.startswith("int8")
                  else T * wl.d // 4 if wl.act.startswith("int2") else T * wl.d // 2)
    rq_bytes = T * wl.d * 2 + code_bytes + 4 * T * (2 if wl.center else 1)
    peaks, peak_kind = load_peaks()
    long_region = elapsed_ms > 1000.0
    bf16_peak = peaks.get("bf16_tflops_sustained" if long_region else "bf16_tflops",
                          peaks["bf16_tflops"])
    fp_gemm = "lloydmax" in wl.act or g64          # fp16 operands on the tensor cores
    rule_peak = bf16_peak * (INT8_PER_BF16 if not fp_gemm else 1.0)
    # the dense tensor-core peak of this GPU for the GEMM's own MMA kind, measured now by the
    # library's peak loop (the GEMM's instruction issued back to back on resident operands)
    loop_kind = "f16" if fp_gemm else "i8"
    tensor_peak, loop_ms = measured_mma_peak(oq, loop_kind, stream)
    hbm_peak = peaks["hbm_gbs"]
    gemm_tops = ops / (max(gm_ms, 1e-9) * 1e-3) / 1e12
    rq_gbs = rq_bytes / (rq_ms * 1e-3) / 1e9
    # captures are of the workload at its own token count (or T = 256 for the single launch)
    tkey = wl.name if T == wl.T else f"{wl.name}@T{T}"
    traffic = ncu_traffic(tkey, "k_gemm")
    traffic_rq = ncu_traffic(tkey, "k_rotate_quant")
    rule_note = (f"{peak_kind} {'sustained' if long_region else 'burst'} bf16 "
                 f"{bf16_peak} TFLOP/s" + (" x 2 (nominal int8/bf16 ratio)"
                                           if not fp_gemm else ""))
    peak_note = (f"tcgen05 kind::{loop_kind} peak loop measured in this run "
                 f"(oq_mma_peak_loop, one CTA pair per two SMs, {loop_ms:.3f} ms)")
    gemm_roof = {"bound": "tensor", "achieved": gemm_tops, "peak": tensor_peak,
                 "unit": "TOPS" if not fp_gemm else "TFLOP/s",
                 "frac": gemm_tops / tensor_peak, "traffic": traffic, "kernel": "k_gemm",
                 "peak_source": peak_note, "ms_per_launch": gm_ms,
                 "peak_rule": rule_peak, "frac_rule": gemm_tops / rule_peak,
                 "peak_rule_source": rule_note}
    rq_roof = {"bound": "hbm", "achieved": rq_gbs, "peak": hbm_peak, "unit": "GB/s",
               "frac": rq_gbs / hbm_peak, "traffic": traffic_rq, "kernel": "k_rotate_quant",
               "peak_source": f"{peak_kind} copy bandwidth", "ms_per_launch": rq_ms,
               "algorithmic_bytes": rq_bytes}
    dominant = gemm_roof if gm_ms >= rq_ms else rq_roof
    other = rq_roof if dominant is gemm_roof else gemm_roof
    shares = {"k_rotate_quant": rq_ms / (rq_ms + gm_ms), "k_gemm": gm_ms / (rq_ms + gm_ms)}
    if fused:
        # one kernel does everything: its HBM floor is reading x and the packed weights and
        # writing y and the workspace's codes (one byte each), scales and means once
        layer_bytes = (T * wl.d * 2 + wl.n_out * wl.d // 2 + wl.n_out * 4 * (2 if wl.center else 1)
                       + T * wl.n_out * 2 + T * wl.d + 4 * T * (2 if wl.center else 1))
        f_gbs = layer_bytes / (rq_ms * 1e-3) / 1e9
        f_tops = ops / (rq_ms * 1e-3) / 1e12
        dominant = {"bound": "hbm", "achieved": f_gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": f_gbs / hbm_peak,
                    "traffic": ncu_traffic(tkey, "k_linear_fused"),
                    "kernel": "k_linear_fused",
                    "peak_source": f"{peak_kind} copy bandwidth", "ms_per_launch": rq_ms,
                    "algorithmic_bytes": layer_bytes}
        other = {"bound": "tensor", "achieved": f_tops, "peak": tensor_peak, "unit": "TOPS",
                 "frac": f_tops / tensor_peak, "kernel": "k_linear_fused",
                 "peak_source": peak_note, "ms_per_launch": rq_ms}
        shares = {"k_linear_fused": 1.0}
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8" if not fp_gemm else "f16",
        "data": "synthetic", "config": config_of(wl, T, world, ring, fused=fused),
        "rotate_quantize_gbs": None if fused else rq_gbs,
        "rotate_quantize_frac_hbm": None if fused else rq_gbs / hbm_peak,
        "gemm_tops": None if fused else gemm_tops,
        "gemm_frac_tensor": None if fused else gemm_tops / tensor_peak,
        "timing": "steps and per-kernel averages replay CUDA graphs of the library's launches",
        "roofline": dominant, "roofline_other": other,
        "kernel_share": shares,
        "e2e": {"value": whole_job_rate(ops, world, e2e_ms) / 1e12, "unit": "TOPS",
                "h2d_bytes_per_step": T * wl.d * 2, "d2h_bytes_per_step": T * wl.n_out * 2,
                "ms_per_step": e2e_ms, "steps": args.e2e_steps},
        "gpu_launches": (1 if fused else 2) * K,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, x_host_bits, w_bits, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    plan.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
