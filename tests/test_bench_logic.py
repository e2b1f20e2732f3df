"""Host-side measurement logic of bench.py (CPU only): which measured peak a
tensor-bound figure is held against, and when recorded ncu counters still
belong to the current kernel sources."""
import json
import os

import bench

PEAKS = {"hbm_gbs": 6551.4, "bf16_tflops": 1636.8, "bf16_tflops_sustained": 1388.9}


def test_short_timed_region_uses_the_burst_peak():
    flops = 5.841155522560e12
    ms = 1.3
    r = bench.tensor_roofline("k", flops, ms, PEAKS, "measured", None, timed_s=0.003)
    burst = PEAKS["bf16_tflops"] * bench.FP4_OVER_BF16
    sust = PEAKS["bf16_tflops_sustained"] * bench.FP4_OVER_BF16
    achieved = flops / (ms * 1e-3) / 1e12
    assert r["regime"].startswith("burst")
    assert abs(r["peak"] - burst) < 0.1
    assert abs(r["frac"] - achieved / burst) < 1e-4
    assert abs(r["frac_of_sustained_peak"] - achieved / sust) < 1e-4
    assert "frac_of_burst_peak" not in r


def test_long_timed_region_uses_the_sustained_peak():
    flops = 5.841155522560e12
    ms = 1.5
    r = bench.tensor_roofline("k", flops, ms, PEAKS, "measured", 123, timed_s=bench.SUSTAINED_S)
    burst = PEAKS["bf16_tflops"] * bench.FP4_OVER_BF16
    sust = PEAKS["bf16_tflops_sustained"] * bench.FP4_OVER_BF16
    achieved = flops / (ms * 1e-3) / 1e12
    assert r["regime"].startswith("sustained")
    assert abs(r["peak"] - sust) < 0.1
    assert abs(r["frac"] - achieved / sust) < 1e-4
    assert abs(r["frac_of_burst_peak"] - achieved / burst) < 1e-4
    assert r["traffic"] == 123
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"


def test_source_hash_ignores_comments_and_blank_lines_only():
    src = {"gemm.cu": "int a;  // one\n\n// two\nint b;\n", "block_quant.cuh": "x", "ptx.cuh": "y",
           "common.h": "z", "runtime.cu": "w"}
    base = bench.source_hash("nvfp4_gemm_kernel", read=lambda n: src[n])
    commented = dict(src, **{"gemm.cu": "int a;  // changed comment\n// another\n\nint b;  // new\n"})
    assert bench.source_hash("nvfp4_gemm_kernel", read=lambda n: commented[n]) == base
    changed = dict(src, **{"gemm.cu": "int a;\nint c;\n"})
    assert bench.source_hash("nvfp4_gemm_kernel", read=lambda n: changed[n]) != base
    other = dict(src, **{"runtime.cu": "v"})
    assert bench.source_hash("nvfp4_gemm_kernel", read=lambda n: other[n]) != base


def test_recorded_traffic_is_reported_only_for_matching_sources():
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    with open(path) as f:
        table = json.load(f)
    for key, entry in table.items():
        if key.startswith("_"):
            continue
        kernel, workload = key.split(":", 1)
        got = bench.profiled_traffic(kernel, workload)
        if entry["source_hash"] == bench.source_hash(kernel):
            assert got == entry["dram_bytes_per_launch"], key
        else:
            assert got is None, key
