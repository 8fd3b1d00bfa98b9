"""Host logic of bench.py: the algorithmic work it divides by, and the recorded DRAM-traffic
figure, which it reports only for the workload, layout and GEMM sources it was captured on."""
import json

import pytest

import bench
import moe_synth


def test_algorithmic_bytes_per_expert():
    """Weights and scales of one touched expert: 3·d·F int8 bytes plus the bf16 scales of
    linear / linear_v ([F] each) and linear_1 ([d]), i.e. 604.1 MB at the Grok-1 shape."""
    w = moe_synth.WORKLOADS["decode"]
    d, F = w.d, w.F
    one = bench.algorithmic_work(w, 0, 1, None)
    two = bench.algorithmic_work(w, 0, 2, None)
    per_expert = (two["up_bytes"] + two["dn_bytes"]) - (one["up_bytes"] + one["dn_bytes"])
    assert per_expert == 3 * d * F + 2 * (2 * F + d)
    assert abs(per_expert / 1e6 - 604.1) < 0.1


def test_algorithmic_work_of_the_routes():
    """Per route: a d-wide bf16 row in and an F-wide bf16 row of H out (up), the H row in and
    an fp32 slot row out (down); 2·d·F FLOPs per matrix."""
    w = moe_synth.WORKLOADS["decode"]
    d, F, T = w.d, w.F, 8
    base = bench.algorithmic_work(w, 0, 7, None)
    work = bench.algorithmic_work(w, T, 7, None)
    R = 2 * T
    assert work["up_bytes"] - base["up_bytes"] == R * d * 2 + R * F * 2
    assert work["dn_bytes"] - base["dn_bytes"] == R * F * 2 + R * d * 4
    assert work["up_flops"] == 2.0 * R * d * F * 2
    assert work["dn_flops"] == 2.0 * R * F * d


def test_block_scales_add_their_bytes():
    w = moe_synth.WORKLOADS["decode"]
    d, F = w.d, w.F
    chan = bench.algorithmic_work(w, 0, 1, None, 0)
    blk = bench.algorithmic_work(w, 0, 1, None, 128)
    assert blk["up_bytes"] - chan["up_bytes"] == 2 * 2 * F * (d // 128 - 1)
    assert blk["dn_bytes"] - chan["dn_bytes"] == 2 * d * (F // 128 - 1)


def test_recorded_traffic_is_keyed(tmp_path, monkeypatch):
    rec = {"decode/packed/up_proj": {"bytes_per_launch": 123, "source_hash": "abc"}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda layout: "abc" if layout == "packed" else "xyz")
    assert bench.recorded_traffic("decode", "packed", "up_proj", False) == 123
    assert bench.recorded_traffic("decode", "packed", "up_proj", True) is None      # resized / other scales
    assert bench.recorded_traffic("decode", "in_out", "up_proj", False) is None     # another kernel
    assert bench.recorded_traffic("prefill", "packed", "up_proj", False) is None    # not recorded
    monkeypatch.setattr(bench, "kernel_source_hash", lambda layout: "changed")
    assert bench.recorded_traffic("decode", "packed", "up_proj", False) is None     # sources changed


def test_source_hash_covers_each_layouts_gemm():
    assert bench.kernel_source_hash("packed") != bench.kernel_source_hash("in_out")
    assert set(bench.GEMM_SOURCES["packed"]) >= {"gemm_ts.cu", "gemm_common.cuh", "ptx.cuh"}


def test_kernel_times_over_regions():
    """The per-kernel times behind the roofline: each kernel's mean launch time per profiled region,
    then the median over the regions (so one region under a different clock does not move it);
    kernels that did not run read 0; launches per step from the region's launch counts."""
    K = 10
    regions = [
        {"up_proj": (100.0, 10), "down_proj": (50.0, 10), "router": (0.0, 0)},
        {"up_proj": (130.0, 10), "down_proj": (52.0, 10), "router": (0.0, 0)},   # a slow region
        {"up_proj": (101.0, 10), "down_proj": (51.0, 10), "router": (0.0, 0)},
    ]
    per_launch, lps = bench.kernel_times_over_regions(regions, K)
    assert per_launch == {"up_proj": 10.1, "down_proj": 5.1, "router": 0.0}
    assert lps == 2.0

