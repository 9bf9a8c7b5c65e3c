"""Multi-rank host logic of bench.py on CPU: gloo, world size 2 (no GPU).

The path shards independent token batches across ranks (weak scaling) with no data-path
collective; what the ranks share is the timing protocol: the step time is the maximum over
ranks and the reported throughput counts the units of every rank.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, local_ms, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(local_ms[rank], world, dist, "cpu")
        rate = bench.whole_job_rate(1000.0, world, t)
        q.put((rank, t, rate))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("local_ms", [(1.5, 2.5), (4.0, 0.25)])
def test_step_time_is_max_over_ranks(local_ms):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    want = max(local_ms)
    for rank, t, rate in got:
        assert t == want                            # every rank sees the slowest rank's time
        assert rate == pytest.approx(1000.0 * world / (want * 1e-3))


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.whole_job_rate(10.0, 1, 2.0) == pytest.approx(5000.0)


def test_ranks_draw_different_inputs_of_the_same_shape():
    import bench
    import synth
    wl = synth.WORKLOADS["tiny"]
    seeds = {bench.input_seed(wl.seed, rank, r) for rank in range(8) for r in range(4)}
    assert len(seeds) == 32
    a = synth.make_x(16, wl.d, mean_var=wl.mean_var, seed=bench.input_seed(wl.seed, 0, 0))
    b = synth.make_x(16, wl.d, mean_var=wl.mean_var, seed=bench.input_seed(wl.seed, 1, 0))
    assert a.shape == b.shape and (a != b).any()


def test_reference_arm_runs_on_rank_zero_only():
    import argparse
    import bench
    import synth
    args = argparse.Namespace(steps=1, warmup=0, gpus=2)
    assert bench.run_reference(args, synth.WORKLOADS["tiny"], rank=1) is None


@pytest.mark.parametrize("name", ["mlp_up_g64", "tiny"])
def test_bench_oracle_leg_is_the_layer_oracle(name):
    # the CPU leg of bench.py (cpu_baseline and --impl reference) computes the layer oracle
    import numpy as np
    import bench
    import oracle
    import synth
    from oracle import weights_g64
    wl, xb, wb = synth.make_inputs(name, T=3)
    x = synth.bf16_to_f64(xb)
    got = bench.oracle_pass(wl, bench.oracle_setup(wl, xb, wb), x)
    plan = oracle.rpbh_plan(wl.d, wl.h, wl.rounds, wl.seed)
    if wl.weights == "int4_g64":
        ref, _, _ = weights_g64.linear_forward_g64(x, synth.bf16_to_f64(wb), plan, wl.h, wl.act,
                                                   wl.center)
    else:
        ref, _, _ = oracle.linear_forward(x, synth.bf16_to_f64(wb), plan, wl.h, wl.act, wl.center)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
