"""Host logic of bench.py on CPU (no GPU): the rules that decide what a bench line may claim.

- A DRAM-traffic figure from an ncu capture is reported only while the kernel's sources are
  byte for byte those it was captured on (sha256 of the files); any edit makes it null.
- The timed steps rotate over input sets that together hold at least twice the L2, so every
  step reads its operands from HBM (at least RING sets, at most 256).
- The algorithmic code bytes per token follow the activation kind: d (8-bit), d/2 (4-bit),
  d/4 (2-bit).
"""
import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    # copy the sources of every kernel that has a traffic entry into a scratch tree
    names = {f for files in bench.KERNEL_SOURCES.values() for f in files}
    for f in names:
        shutil.copy(bench.csrc(f), tmp_path / f)
    monkeypatch.setattr(bench, "csrc", lambda name: str(tmp_path / name))
    # same bytes: every entry's figure is reported
    for key, entry in bench.NCU_TRAFFIC.items():
        assert bench.ncu_traffic(*key) == entry["bytes"], key
    # one byte appended to a file that only the rotate-quantize entry depends on
    with open(tmp_path / "k_rotate_quant.cu", "ab") as fh:
        fh.write(b"\n")
    assert bench.ncu_traffic("dit_w4a8", "k_rotate_quant") is None
    assert bench.ncu_traffic("dit_w4a8", "k_gemm") == bench.NCU_TRAFFIC[("dit_w4a8", "k_gemm")]["bytes"]
    # a file two kernels share (the PTX wrappers) invalidates both
    with open(tmp_path / "ptx.cuh", "ab") as fh:
        fh.write(b"\n")
    assert bench.ncu_traffic("dit_w4a8", "k_gemm") is None
    assert bench.ncu_traffic("dit_w4a8@T256", "k_linear_fused") is None


def test_traffic_entries_name_known_kernels_and_positive_bytes():
    for (workload, kernel), entry in bench.NCU_TRAFFIC.items():
        assert workload.split("@")[0] in synth.WORKLOADS
        assert entry.get("sources", kernel) in bench.KERNEL_SOURCES
        assert kernel in bench.KERNEL_SOURCES or "sources" in entry
        assert isinstance(entry["bytes"], int) and entry["bytes"] > 0
        assert len(entry["sha"]) == 64
    assert bench.ncu_traffic("no_such_workload", "k_gemm") is None


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
@pytest.mark.parametrize("T", [1, 64, 256, 4096])
def test_input_ring_holds_twice_the_l2(name, T):
    wl = synth.WORKLOADS[name]
    ring = bench.ring_size(wl, T, bench.L2_BYTES)
    assert bench.RING <= ring <= 256
    if ring < 256:
        assert ring * bench.set_bytes(wl, T) >= 2 * bench.L2_BYTES
        # and no set more than needed
        assert ring == bench.RING or (ring - 1) * bench.set_bytes(wl, T) < 2 * bench.L2_BYTES


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
def test_set_bytes_counts_the_kind_s_code_width(name):
    wl = synth.WORKLOADS[name]
    T = 128
    per_code = {"int8": 8, "int4": 4, "int2": 2}[wl.act[:4]]
    fixed = T * wl.d * 2 + wl.n_out * wl.d // 2 + 12 * wl.n_out + 8 * T + T * wl.n_out * 2
    assert bench.set_bytes(wl, T) - fixed == T * wl.d * per_code // 8


def test_config_names_the_workload_and_path():
    wl = synth.WORKLOADS["dit_w4a8"]
    c = bench.config_of(wl, 4096, 1)
    assert c["workload"] == "dit_w4a8" and c["T"] == 4096
    assert (c["d_in"], c["d_out"], c["h"], c["rounds"]) == (3072, 3072, 1024, 1)
    assert c["parallelism"] == "replicas" and "path" not in c
    assert "L2" in c["l2"]
    assert bench.config_of(wl, 256, 1, fused=True)["path"].startswith("single launch")
    assert bench.config_of(wl, 4096, 2)["parallelism"].startswith("dp2")


def test_single_launch_kinds():
    # the kinds the single-launch layer takes: INT8 absmax and the two INT4 scales
    assert set(bench.FUSED_ACTS) == {"int8_absmax", "int4_absmax", "int4_percentile"}
    import w4a8_ptq_linear_b200 as oq
    assert set(bench.FUSED_ACTS) <= set(oq.ACT_KINDS)


def test_input_seeds_differ_across_ranks_and_sets():
    seeds = {bench.input_seed(0, rank, r) for rank in range(8) for r in range(256)}
    assert len(seeds) == 8 * 256
