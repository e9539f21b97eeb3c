"""The algorithmic FLOP and byte counts behind bench.py's roofline fractions, checked on small
cases against the definitions written out by hand: each operand once, the rows that are
computed (contiguous: valid rows; masked: rows below masked_m), the groups touched, an FP4 B at
half a byte per element, and t_roof = max(FLOPs / P_fp8, bytes / BW)."""
from __future__ import annotations

import numpy as np
import pytest

import bench
import workloads


def test_dense_counts():
    c = workloads.dense(64, 256, 384, seed=1)
    g = bench.Gemm("dense", c, "d")
    assert g.flops == 2.0 * 64 * 256 * 384
    kb, nb = 3, 2
    assert g.bytes == 64 * 384 + 256 * 384 + 2 * 64 * 256 + 4 * 64 * kb + 4 * nb * kb


def test_dense_fp4_halves_b():
    c = workloads.dense(64, 256, 384, seed=1)
    g8 = bench.Gemm("dense", c, "d")
    g4 = bench.Gemm("dense", workloads.with_fp4_b(c, seed=2), "d fp4", fp4=True)
    assert g8.flops == g4.flops
    assert g8.bytes - g4.bytes == 256 * 384 // 2


def test_contiguous_counts_valid_rows_and_touched_groups():
    c = workloads.contiguous(G=4, N=128, K=256, seed=3, counts=[5, 0, 130, 128])
    g = bench.Gemm("contiguous", c, "c")
    m_valid = 5 + 130 + 128
    m_rows = c.M_total                       # 128 + 0 + 256 + 128 = 512
    assert m_rows == 512
    assert g.flops == 2.0 * m_valid * 128 * 256
    kb = 2
    assert g.bytes == (m_valid * 256 + 128 * 256 * 3 + 2 * m_valid * 128 + 4 * m_rows * kb
                       + 4 * 1 * kb * 3 + 4 * m_rows)


def test_masked_counts_rows_below_masked_m():
    c = workloads.masked(G=3, M_max=64, N=256, K=128, seed=4, masked_m=[10, 0, 64])
    g = bench.Gemm("masked", c, "m")
    assert g.flops == 2.0 * 74 * 256 * 128
    assert g.bytes == 74 * 128 + 256 * 128 * 2 + 2 * 74 * 256 + 4 * 74 * 1 + 4 * 2 * 1 * 2


def test_roofline_bound_and_fraction():
    c = workloads.dense(4096, 4096, 4096, seed=5)
    g = bench.Gemm("dense", c, "big")
    peaks = dict(hbm_gbs=6000.0, bf16_tflops=1500.0, bf16_tflops_sustained=1400.0, source="test")
    p_fp8 = 1500.0 * bench.FP8_PER_BF16 * 1e12
    t_roof = max(g.flops / p_fp8, g.bytes / 6000e9)
    r = bench.roofline(g, 2 * t_roof, peaks)
    assert r["bound"] == "tensor"
    assert r["frac"] == pytest.approx(0.5)
    assert r["tflops"] == pytest.approx(g.flops / (2 * t_roof) / 1e12)
    small = bench.Gemm("dense", workloads.dense(64, 4096, 4096, seed=6), "small")
    assert bench.roofline(small, 1e-3, peaks)["bound"] == "hbm"


def test_quant_and_swiglu_bytes():
    assert bench.quant_bytes(8, 256) == 8 * 256 * 2 + 8 * 256 + 4 * 8 * 2
    assert bench.swiglu_bytes(8, 256) == 8 * 512 * 2 + 8 * 256 + 4 * 8 * 2


def test_per_config_sums_times_and_roofline():
    """per_config: TFLOPS and GB/s over a configuration's summed times, and the fraction as
    summed roofline time over summed time (graph fraction only when every GEMM has one)."""
    shapes = [
        dict(config=2, us=10.0, roof_us=5.0, tflops=1.0, gbs=100.0, bound="hbm", graph_us=8.0),
        dict(config=2, us=30.0, roof_us=15.0, tflops=3.0, gbs=300.0, bound="tensor"),
        dict(config=4, us=20.0, roof_us=16.0, tflops=2.0, gbs=500.0, bound="hbm", graph_us=18.0),
    ]
    pc = {e["config"]: e for e in bench.per_config(shapes)}
    assert pc[2]["us"] == 40.0 and pc[2]["frac"] == pytest.approx(0.5)
    assert pc[2]["tflops"] == pytest.approx((10 * 1.0 + 30 * 3.0) / 40)
    assert pc[2]["gbs"] == pytest.approx((10 * 100 + 30 * 300) / 40)
    assert "graph_frac" not in pc[2] and pc[2]["bound"] == ["hbm", "tensor"]
    assert pc[4]["graph_frac"] == pytest.approx(16.0 / 18.0)


def test_traffic_reported_only_for_unchanged_kernel_sources(monkeypatch):
    fp = bench.kernel_source_fingerprint()
    assert len(fp) == 16 and fp == bench.kernel_source_fingerprint()
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "k same", (123, fp))
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "k stale", (456, "0" * 16))
    assert bench.measured_traffic("k same")[0] == 123
    assert bench.measured_traffic("k stale")[0] is None
    assert bench.measured_traffic("k unknown")[0] is None
    assert bench.measured_traffic("k stale", 789)[0] == 789


def test_library_stick_reports_why_when_the_child_fails(monkeypatch):
    """The library measuring stick runs in a child process; when that process fails (no GPU,
    no library) the line carries the reason and no numbers, and a child's JSON is passed on."""
    import subprocess
    import types

    def failing(*a, **k):
        return types.SimpleNamespace(returncode=1, stdout="", stderr="ModuleNotFoundError: no vllm\n")
    monkeypatch.setattr(subprocess, "run", failing)
    r = bench.library_stick([(8192, 7168, 18432)])
    assert r["unavailable"] == "ModuleNotFoundError: no vllm" and "shapes" not in r

    def raising(*a, **k):
        raise subprocess.TimeoutExpired(cmd="bench.py", timeout=300)
    monkeypatch.setattr(subprocess, "run", raising)
    assert "TimeoutExpired" in bench.library_stick([(64, 2112, 7168)])["unavailable"]

    seen = {}

    def ok(cmd, **k):
        seen["arg"] = cmd[cmd.index("--library-stick") + 1]
        return types.SimpleNamespace(returncode=0, stderr="",
                                     stdout='noise\n{"library": "x", "shapes": [{"shape": "1x2x3"}]}\n')
    monkeypatch.setattr(subprocess, "run", ok)
    r = bench.library_stick([(8192, 7168, 18432), (64, 2112, 7168)])
    assert seen["arg"] == "8192,7168,18432;64,2112,7168"
    assert r["shapes"][0]["shape"] == "1x2x3"
