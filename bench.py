#!/usr/bin/env python
"""Benchmark of the FP8 block-scaled NT GEMM library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload sweep|small|contiguous|masked|prefill|dense|quant|swiglu]
                    [--fp4]

Prints ONE JSON line on rank 0.  A "step" is one pass of the whole hot path over one batch of
synthetic input: for the default workload ("all"), the nineteen GEMMs of the five workload
configurations, each GEMM once:
  1. dense 128 x 256 x 512, A and B ~ N(0,1);
  2. the dense sweep, M in {64, 128, 4096} x (N, K) in {(2112,7168), (24576,1536),
     (7168,16384), (4096,7168), (7168,2048)}, A ~ N(0,1), B ~ N(0,0.02^2) (15 GEMMs);
  3. the contiguous grouped MoE GEMM, G = 8, per-expert counts U[128, 1024] padded to 128,
     N = 4096, K = 7168;
  4. the masked grouped MoE GEMM, G = 32, M_max = 256, masked_m U[0, 256], N = 4096, K = 7168;
  5. the prefill GEMM 8192 x 7168 x 18432 with 1 % x50 outliers in A;
all with fp32 scales per 1x128 tile of A and per 128x128 block of B.  `per_shape` has one
entry per GEMM and `per_config` one per configuration.  Inputs are resident in HBM.  Each timed step is one CUDA event pair on the
launching stream around the step's GEMMs, enqueued back to back as a user would (programmatic
dependent launch lets each kernel's set-up overlap the previous one's tail); the step is
enqueued behind a bounded sleep kernel so that host latency never falls inside the bracket.  L2
is flushed (a 256 MiB write) before every step, outside the bracket, and the step's own working
set exceeds L2.  A second pass of the same steps brackets every GEMM with its own events for the
per-shape figures and the roofline of the dominant kernel.

`value` is the aggregate FP8 TFLOPS of the step (sum of 2*M*N*K over its GEMMs / device time of
the step), summed over ranks (each rank runs its own copy of the step: weak scaling, no
collective on the data path).  `e2e` is the same metric through the Python binding with host
buffers: pinned host -> device copies of every input, the GEMMs, and the device -> host copy of
every output inside the timed region.  `--impl reference` times the CPU oracle on a bounded
sample of the same workload on this machine's cores.  `--fp4` makes B of every GEMM a packed
FP4 (E2M1) operand and runs the FP8 x FP4 entries on the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "FP8 TFLOPS and GB/s per shape at 1 B200; fraction of FP8-peak/HBM roofline"
UNIT = "TFLOPS"
L2_FLUSH_BYTES = 256 << 20
FP8_PER_BF16 = 2.0  # nominal dense FP8 / BF16 tensor ratio on B200 (4.5 / 2.25 PFLOP/s)
SPEC_FP8_TFLOPS = 4500.0  # B200 dense FP8 tensor peak (data sheet)
SPEC_HBM_GBS = 8000.0     # B200 HBM3e bandwidth (data sheet)

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant kernel
# of a workload, from one ncu capture (summaries under profiles/), with the fingerprint of the
# kernel sources it was taken on (`kernel_source_fingerprint`).  `roofline.traffic` reports the
# figure only while the sources still have that fingerprint, and null once a kernel changed
# since the counters were taken; --traffic-bytes overrides it.
MEASURED_TRAFFIC = {
    "dense 8192x7168x18432": (1094379776 + 112736512, "358a90c0e22a9612"),   # CTA pair BN 256
    "dg_quantize_1x128_kernel 8192x7168": (117451520 + 9024512, None),
    "dg_swiglu_quantize_1x128_kernel 16384x4096": (134243072 + 7325696, None),
}


def kernel_source_fingerprint() -> str:
    """sha256 (first 16 hex digits) of the library's CUDA sources and its header."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fp8_block_scaled_tma_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    with open(os.path.join(ROOT, "include", "dg.h"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(name: str, override=None):
    """(bytes per launch or None, note) for the dominant kernel `name`."""
    if override:
        return override, "--traffic-bytes"
    if name not in MEASURED_TRAFFIC:
        return None, "no ncu capture of this kernel"
    value, fp = MEASURED_TRAFFIC[name]
    if fp is not None and fp != kernel_source_fingerprint():
        return None, "the kernel sources changed since the ncu capture"
    return value, f"ncu capture, kernel sources {fp or 'not fingerprinted'}"


# ---- workload description ---------------------------------------------------------------------

class Gemm:
    """One GEMM of a step: its kind, sizes, FLOPs and algorithmic bytes."""

    def __init__(self, kind: str, case, name: str, fp4: bool = False, config: int = 0):
        self.kind, self.case, self.name, self.fp4, self.config = kind, case, name, fp4, config
        self._oracle_b = None
        c = case
        if kind == "dense":
            M, N, K, groups, m_valid, m_rows = c.M, c.N, c.K, 1, c.M, c.M
        elif kind == "contiguous":
            M, N, K = c.M_total, c.N, c.K
            m_valid, m_rows = int(c.counts.sum()), c.M_total
            groups = int(np.count_nonzero(c.counts))
        else:
            M, N, K = c.M_max, c.N, c.K
            m_valid, m_rows = int(c.masked_m.sum()), int(c.masked_m.sum())
            groups = int(np.count_nonzero(c.masked_m))
        kb, nb = K // 128, -(-N // 128)
        self.flops = 2.0 * m_valid * N * K
        # each operand once: A rows that are computed, B of every group touched, D, the scales,
        # and the int32 row indices of the contiguous layout
        # (a packed FP4 B is half a byte per element)
        b_bytes = N * K * groups // (2 if fp4 else 1)
        self.bytes = (m_valid * K + b_bytes + 2 * m_valid * N + 4 * m_rows * kb
                      + 4 * nb * kb * groups + (4 * M if kind == "contiguous" else 0))
        self.shape = dict(kind=kind, M=M, N=N, K=K, G=getattr(c, "G", 1), M_valid=m_valid)
        if config:
            self.shape["config"] = config

    def oracle_b(self):
        """B as the oracle takes it: e4m3 codes (an FP4 B expanded once by the oracle)."""
        if not self.fp4:
            return self.case.b
        if self._oracle_b is None:
            import oracle
            self._oracle_b = oracle.e2m1_to_e4m3(self.case.b)
        return self._oracle_b


def build_workload(name: str, shape=None, fp4: bool = False):
    """The GEMMs of one step.  fp4: every B becomes a packed E2M1 operand (seeded, with its own
    128x128 block scales) and the step runs the FP8 x FP4 entries."""
    gemms, desc = _build_workload(name, shape)
    if not fp4:
        return gemms, desc
    out = []
    for i, g in enumerate(gemms):
        out.append(Gemm(g.kind, workloads.with_fp4_b(g.case, seed=7000 + i), g.name + " fp4", fp4=True,
                        config=g.config))
    return out, desc.replace("B~N(0,0.02)", "B packed FP4 E2M1 (uniform codes, 128x128 fp32 block scales)") \
        + "; FP8 x FP4"


CONFIG_NAMES = {1: "dense 128x256x512", 2: "dense sweep (15 shapes)", 3: "contiguous G=8",
                4: "masked G=32", 5: "prefill 8192x7168x18432"}


def _build_workload(name: str, shape=None):
    if name == "all":
        parts = [("small", 1), ("sweep", 2), ("contiguous", 3), ("masked", 4), ("prefill", 5)]
        gemms, descs = [], []
        for part, cfg in parts:
            gs, d = _build_workload(part)
            for g in gs:
                g.config = cfg
                g.shape["config"] = cfg
            gemms += gs
            descs.append(f"({cfg}) {d}")
        return gemms, "the five configurations, each GEMM once per step: " + "; ".join(descs)
    if name == "dense":
        M, N, K = shape
        c = workloads.dense(M, N, K, seed=6000, a_std=1.0, b_std=0.02)
        return [Gemm("dense", c, f"dense {M}x{N}x{K}")], \
            f"dense FP8 NT GEMM M={M} N={N} K={K}, A~N(0,1), B~N(0,0.02)"
    if name == "sweep":
        gemms = []
        for i, (M, N, K) in enumerate(workloads.sweep_shapes()):
            gemms.append(Gemm("dense", workloads.sweep_case(i), f"dense {M}x{N}x{K}"))
        desc = ("dense FP8 NT GEMM sweep, M in {64,128,4096} x (N,K) in {(2112,7168),(24576,1536),"
                "(7168,16384),(4096,7168),(7168,2048)}; A~N(0,1), B~N(0,0.02); fp32 scales per 1x128 "
                "A tile and 128x128 B block; bf16 out")
        return gemms, desc
    if name == "small":
        c = workloads.small_dense()
        return [Gemm("dense", c, "dense 128x256x512")], "dense FP8 NT GEMM M=128 N=256 K=512, A,B~N(0,1)"
    if name == "contiguous":
        c = workloads.contiguous_case()
        return [Gemm("contiguous", c, f"contiguous G=8 M_total={c.M_total} N=4096 K=7168")], \
            ("contiguous grouped MoE GEMM, G=8, per-expert counts U[128,1024] padded to 128, "
             "N=4096, K=7168, B~N(0,0.02)")
    if name == "masked":
        c = workloads.masked_case()
        return [Gemm("masked", c, "masked G=32 M_max=256 N=4096 K=7168")], \
            ("masked grouped MoE GEMM, G=32, M_max=256, masked_m U[0,256], expected_m=128, "
             "N=4096, K=7168, B~N(0,0.02)")
    if name == "prefill":
        c = workloads.prefill_case()
        return [Gemm("dense", c, "dense 8192x7168x18432")], \
            "dense FP8 NT GEMM M=8192 N=7168 K=18432, A~N(0,1) with 1% x50 outliers, B~N(0,0.02)"
    raise SystemExit(f"unknown workload {name}")


# ---- peaks and roofline ---------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def roofline(g: Gemm, seconds: float, peaks) -> dict:
    """Per-shape figures: `frac` against the measured denominators (2 x the measured bf16 GEMM
    for FP8, the measured copy bandwidth for HBM), `frac_spec` against the data-sheet ones."""
    fp8_peak = peaks["bf16_tflops"] * FP8_PER_BF16 * 1e12
    bw = peaks["hbm_gbs"] * 1e9
    t_flop, t_mem = g.flops / fp8_peak, g.bytes / bw
    t_spec = max(g.flops / (SPEC_FP8_TFLOPS * 1e12), g.bytes / (SPEC_HBM_GBS * 1e9))
    bound = "tensor" if t_flop >= t_mem else "hbm"
    return dict(name=g.name, **g.shape, us=seconds * 1e6, tflops=g.flops / seconds / 1e12,
                gbs=g.bytes / seconds / 1e9, bound=bound, roof_us=max(t_flop, t_mem) * 1e6,
                frac=max(t_flop, t_mem) / seconds, frac_spec=t_spec / seconds)


def measure_cublas_fp8(n: int = 8192, reps: int = 10):
    """A measuring stick for the FP8 tensor peak on this GPU: torch._scaled_mm (cuBLASLt) on an
    n x n x n e4m3 GEMM with per-tensor scales, median of `reps` event-timed runs after
    warm-up.  Never on the product path.  Returns TFLOP/s, or None where unsupported."""
    try:
        g = torch.Generator(device="cuda")
        g.manual_seed(7)
        a = torch.randn(n, n, device="cuda", generator=g).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device="cuda", generator=g).to(torch.float8_e4m3fn)
        one = torch.ones((), device="cuda")
        f = lambda: torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        for _ in range(3):
            f()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e-3)
        return 2.0 * n ** 3 / statistics.median(ts) / 1e12
    except Exception:  # an older torch or cuBLAS without FP8: report nothing
        return None


LIBRARY_STICK = "vLLM cutlass_scaled_mm: CUTLASS block-scaled FP8 GEMM (1x128 A scales, 128x128 B scales)"


def library_stick(shapes, reps: int = 10) -> list:
    """A measuring stick for the same computation from a library: vLLM's cutlass_scaled_mm with
    DeepSeek-style block scales, on seeded inputs of each (M, N, K), timed beside this library's
    dense GEMM on the same inputs (256 MiB L2 flush and a short sleep before every run, median
    of `reps` event-timed runs after warm-up), with the largest difference between the two
    outputs relative to |ours| + 1.  Runs in a child process (`--library-stick`) so that the
    library's import cannot touch this process; never on the product path."""
    import subprocess
    arg = ";".join(f"{m},{n},{k}" for m, n, k in shapes)
    try:
        r = subprocess.run([sys.executable, os.path.abspath(__file__), "--library-stick", arg,
                            "--steps", str(reps), "--warmup", "3"],
                           capture_output=True, text=True, timeout=300)
        lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
        if r.returncode != 0 or not lines:
            tail = (r.stderr or r.stdout).strip().splitlines()[-1:] or ["no output"]
            return dict(library=LIBRARY_STICK, unavailable=tail[0][:200])
        return json.loads(lines[-1])
    except Exception as e:  # no such library, or it failed: report why, measure nothing
        return dict(library=LIBRARY_STICK, unavailable=f"{type(e).__name__}: {e}"[:200])


def run_library_stick(arg: str, reps: int) -> dict:
    """Child side of library_stick."""
    import vllm._custom_ops as ops  # imported here only: the measuring stick's library

    import fp8_block_scaled_tma_b200 as dg
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def timed(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            torch.cuda._sleep(200000)
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        return statistics.median(ts)

    out = []
    for item in arg.split(";"):
        M, N, K = (int(x) for x in item.split(","))
        g = torch.Generator(device="cuda")
        g.manual_seed(M * 7 + N * 3 + K)
        a = (torch.randn(M, K, device="cuda", generator=g) * 0.5).to(torch.float8_e4m3fn)
        b = (torch.randn(N, K, device="cuda", generator=g) * 0.5).to(torch.float8_e4m3fn)
        kb, nb = K // 128, (N + 127) // 128
        sa = torch.rand(M, kb, device="cuda", generator=g) + 0.5
        sb = torch.rand(nb, kb, device="cuda", generator=g) + 0.5
        d = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        sfa = dg.sfa_mn_major(sa)
        ours = lambda: dg.dg_gemm_fp8_fp8_bf16_nt(a.view(torch.uint8), sfa, b.view(torch.uint8), sb, d)
        # the library's layouts: B as [K, N] column-major, A scales [M, K/128] M-contiguous,
        # B scales [K/128, N/128] K-contiguous
        sa_l = sa.t().contiguous().t()
        theirs = lambda: ops.cutlass_scaled_mm(a, b.t(), sa_l, sb.t(), torch.bfloat16)
        us_ours = timed(ours)
        ref = d.float()
        us_lib = timed(theirs)
        diff = ((theirs().float() - ref).abs() / (ref.abs() + 1.0)).max().item()
        fl = 2.0 * M * N * K
        out.append(dict(shape=f"{M}x{N}x{K}", ours_us=us_ours, ours_tflops=fl / us_ours / 1e6,
                        library_us=us_lib, library_tflops=fl / us_lib / 1e6,
                        speedup=us_lib / us_ours, max_rel_diff=diff))
    return dict(library=LIBRARY_STICK, shapes=out)


def back_to_back(dg, dev, flush, gate_cycles: int, reps: int = 10) -> dict:
    """The whole step enqueued back to back (no event between GEMMs), L2 flushed before it,
    timed by one event pair: with programmatic dependent launch off and on.  Each kernel's
    on-chip set-up can then overlap the previous kernel's tail."""
    stream = torch.cuda.current_stream()
    out = dict(gemms=len(dev))
    for key, on in (("pdl_off_ms", False), ("pdl_on_ms", True)):
        prev = dg.set_pdl(on)
        ts = []
        for r in range(reps + 2):
            torch.cuda._sleep(gate_cycles)
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for d in dev:
                d.launch(stream)
            e1.record(stream)
            stream.synchronize()
            ts.append(e0.elapsed_time(e1))
        dg.set_pdl(prev)
        out[key] = statistics.mean(ts[2:])
    return out


def graph_times(dev, flush, reps: int = 20):
    """Per-launch device time of each GEMM inside a CUDA graph of `reps` (L2 flush, GEMM) pairs,
    minus a graph of `reps` flushes alone: the launch-latency-free time of a cold-L2 launch."""
    def timed(graph):
        graph.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e-3)
        return statistics.median(ts)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    base = torch.cuda.CUDAGraph()
    with torch.cuda.graph(base, stream=side):
        for _ in range(reps):
            flush.fill_(1)
    t_flush = timed(base)
    out = []
    for d in dev:
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=side):
            for _ in range(reps):
                flush.fill_(1)
                d.launch()
        out.append(max(0.0, (timed(gr) - t_flush) / reps))
        del gr
    del base
    return out


# ---- clocks ---------------------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a background thread."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                mask = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return dict(sm_mhz=None, sm_max_mhz=self.max_mhz, reasons=sorted(self.reasons), samples=0)
        return dict(sm_mhz=float(statistics.median(self.samples)), sm_max_mhz=self.max_mhz,
                    reasons=sorted(self.reasons - {"gpu_idle"}), samples=len(self.samples))


# ---- multi-rank aggregation ---------------------------------------------------------------------

def max_over_ranks(seconds: float, world: int, device: str) -> float:
    """The slowest rank's device time: every rank runs its own copy of the step (weak scaling),
    so the job is done when the last rank is."""
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_step: float, steps: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the FLOPs all ranks did over the slowest rank's time."""
    return world * flops_per_step * steps / max_seconds / 1e12


# ---- our arm ------------------------------------------------------------------------------------

class DeviceGemm:
    """Device-resident inputs and output of one GEMM, and the launch through the binding."""

    def __init__(self, dg, g: Gemm):
        self.g = g
        c = g.case
        self.a = torch.from_numpy(np.ascontiguousarray(c.a)).cuda()
        self.b = torch.from_numpy(np.ascontiguousarray(c.b)).cuda()
        self.sfa = dg.sfa_mn_major(torch.from_numpy(c.sa).cuda())
        self.sfb = torch.from_numpy(c.sb).cuda()
        self.extra = None
        if g.kind == "dense":
            self.d = torch.empty(c.M, c.N, dtype=torch.bfloat16, device="cuda")
        elif g.kind == "contiguous":
            self.d = torch.empty(c.M_total, c.N, dtype=torch.bfloat16, device="cuda")
            self.extra = torch.from_numpy(c.m_indices).cuda()
        else:
            self.d = torch.empty(c.G, c.M_max, c.N, dtype=torch.bfloat16, device="cuda")
            self.extra = torch.from_numpy(c.masked_m).cuda()
        self.dg = dg

    def tensors_in(self):
        t = [self.a, self.sfa, self.b, self.sfb]
        if self.extra is not None:
            t.append(self.extra)
        return t

    def launch(self, stream=None):
        dg, c = self.dg, self.g.case
        if self.g.fp4:
            if self.g.kind == "dense":
                dg.dg_gemm_fp8_fp4_bf16_nt(self.a, self.sfa, self.b, self.sfb, self.d, stream=stream)
            elif self.g.kind == "contiguous":
                dg.dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous(self.a, self.sfa, self.b, self.sfb,
                                                                self.d, self.extra, stream=stream)
            else:
                dg.dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked(self.a, self.sfa, self.b, self.sfb,
                                                            self.d, self.extra, c.expected_m,
                                                            stream=stream)
        elif self.g.kind == "dense":
            dg.dg_gemm_fp8_fp8_bf16_nt(self.a, self.sfa, self.b, self.sfb, self.d, stream=stream)
        elif self.g.kind == "contiguous":
            dg.dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(self.a, self.sfa, self.b, self.sfb,
                                                            self.d, self.extra, stream=stream)
        else:
            dg.dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(self.a, self.sfa, self.b, self.sfb, self.d,
                                                        self.extra, c.expected_m, stream=stream)


def run_ours(args, rank, world, local_rank):
    import fp8_block_scaled_tma_b200 as dg

    torch.cuda.set_device(local_rank)
    gemms, desc = build_workload(args.workload, args.shape, args.fp4)
    if args.block_n or args.stages or args.splits:
        dg.set_config_override(args.block_n, args.stages, args.splits)
    if args.family:
        dg.set_kernel_family(args.family)
    dev = [DeviceGemm(dg, g) for g in gemms]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    n = len(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    gate = [2_000_000]  # GPU cycles the stream is held so the host can enqueue the whole step

    def gated(enqueue):
        # a bounded sleep kernel holds the stream while the host enqueues the step, so no host
        # latency falls inside an event bracket; then the L2 flush (outside the brackets)
        torch.cuda._sleep(gate[0])
        flush.fill_(1)
        t0 = time.perf_counter()
        enqueue()
        host = time.perf_counter() - t0
        stream.synchronize()
        if host * 1.9e9 * 1.5 > gate[0]:
            gate[0] = int(host * 1.9e9 * 3)

    def step():
        """One step as a user runs it: the GEMMs back to back, one event pair around them."""
        def enqueue():
            ev[0].record(stream)
            for d in dev:
                d.launch(stream)
            ev[n].record(stream)
        gated(enqueue)
        return ev[0].elapsed_time(ev[n]) * 1e-3

    def step_per_gemm():
        """The same step with an event pair around every GEMM (per-shape and roofline figures;
        the events between kernels cost each boundary its launch overlap)."""
        def enqueue():
            for i, d in enumerate(dev):
                ev[i].record(stream)
                d.launch(stream)
            ev[n].record(stream)
        gated(enqueue)
        return [ev[i].elapsed_time(ev[i + 1]) * 1e-3 for i in range(n)]

    for _ in range(args.warmup):
        step()
        step_per_gemm()
    launch_info = dg.get_last_launch()
    if dg.poll_device_error(stream) != 0:
        raise RuntimeError("device error during warm-up")

    # the timed steps: whole-step device time
    step_times = []
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for _ in range(args.steps):
            step_times.append(step())
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    total = sum(step_times)  # device seconds over the timed steps
    total_max = max_over_ranks(total, world, "cuda")

    # per-GEMM breakdown (not part of `value`): the same number of steps with per-GEMM brackets
    per = [[] for _ in range(n)]
    for _ in range(args.steps):
        for i, t in enumerate(step_per_gemm()):
            per[i].append(t)
    if dg.poll_device_error(stream) != 0:
        raise RuntimeError("device error during the timed steps")

    flops_step = sum(g.flops for g in gemms)
    bytes_step = sum(g.bytes for g in gemms)
    value = aggregate_tflops(flops_step, args.steps, world, total_max)
    peaks = load_peaks()
    shapes = [roofline(g, statistics.mean(p), peaks) for g, p in zip(gemms, per)]
    if not args.no_graph:
        # launch-latency-bound shapes (memory-bound, a few microseconds): add the in-graph time
        idx = [i for i, sh in enumerate(shapes) if sh["bound"] == "hbm"]
        if idx:
            gt = graph_times([dev[i] for i in idx], flush)
            for i, t in zip(idx, gt):
                if t > 0:
                    shapes[i].update(graph_us=t * 1e6, graph_frac=shapes[i]["roof_us"] * 1e-6 / t)
        if dg.poll_device_error(stream) != 0:
            raise RuntimeError("device error during the graph timing")
    if not args.no_graph:
        b2b = back_to_back(dg, dev, flush, gate[0])
        if dg.poll_device_error(stream) != 0:
            raise RuntimeError("device error during the back-to-back timing")
    else:
        b2b = None
    dom = max(range(n), key=lambda i: sum(per[i]))
    dsh = shapes[dom]
    if dsh["bound"] == "tensor":
        peak = peaks["bf16_tflops"] * FP8_PER_BF16
        roof = dict(bound="tensor", achieved=dsh["tflops"], peak=peak, unit="TFLOP/s",
                    frac=dsh["tflops"] / peak,
                    peak_source=f"{peaks['source']} bf16 burst x{FP8_PER_BF16:g} (nominal FP8/BF16 ratio)")
    else:
        peak = peaks["hbm_gbs"]
        roof = dict(bound="hbm", achieved=dsh["gbs"], peak=peak, unit="GB/s",
                    frac=dsh["gbs"] / peak, peak_source=f"{peaks['source']} HBM copy")
    traffic, traffic_note = measured_traffic(dsh["name"], args.traffic_bytes)
    roof.update(kernel=dsh["name"], traffic=traffic, traffic_unit="bytes/launch",
                traffic_source=traffic_note, frac_spec=dsh["frac_spec"],
                launches_timed=args.steps)
    if rank == 0 and not args.no_cublas:
        # context only: what cuBLAS reaches on an FP8 GEMM on this GPU
        roof["cublas_fp8_tflops_8192"] = measure_cublas_fp8()

    out = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps,
               warmup=args.warmup, ms_per_step=total_max / args.steps * 1e3,
               higher_is_better=True, scaling="weak", vs_baseline=None,
               dtype="e4m3 x e2m1 -> f32" if args.fp4 else "e4m3 x e4m3 -> f32",
               data="synthetic",
               config=bench_config(desc, n, world),
               gbs=world * bytes_step * args.steps / total_max / 1e9,
               roofline=roof, per_shape=shapes, per_config=per_config(shapes),
               back_to_back=b2b, gpu_launches=n * args.steps,
               clocks=clk.summary(), last_launch=launch_info)

    # e2e through the public API with host buffers
    if not args.no_e2e:
        out["e2e"] = run_e2e(dg, dev, gemms, args, world)
    if rank == 0 and world == 1 and not args.no_library_stick:
        big = sorted(shapes, key=lambda sh: -sh["us"])
        picks = [(sh["M"], sh["N"], sh["K"]) for sh in big if sh["kind"] == "dense"][:1]
        picks += [(sh["M"], sh["N"], sh["K"]) for sh in big
                  if sh["kind"] == "dense" and sh["M"] <= 128 and (sh["M"], sh["N"], sh["K"]) not in picks][:1]
        if picks:
            out["library_stick"] = library_stick(picks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(gemms, budget_s=args.cpu_seconds)
    return out


def bench_config(desc: str, n_gemms: int, world: int) -> dict:
    """The `config` of the JSON line; both arms print the same one for a workload."""
    return dict(workload=desc, gemms_per_step=n_gemms,
                l2="256 MiB write before every step; step working set > L2 (126 MB)",
                timing="value: one CUDA event pair per step on the launching stream around the "
                       "step's GEMMs enqueued back to back (programmatic dependent launch on), the "
                       "step enqueued behind a bounded sleep kernel and the L2 flush outside the "
                       "bracket; per_shape and roofline: a second pass of the same steps with an "
                       "event pair around every GEMM",
                parallelism=f"replicas x{world}" if world > 1 else "single GPU")


def per_config(shapes) -> list:
    """Per workload configuration: its GEMMs' summed event times, TFLOPS and algorithmic GB/s,
    and the fraction of its roofline (summed roofline time / summed time), also in a CUDA
    graph where every GEMM of the configuration has a graph time."""
    out = []
    for cfg in sorted({sh.get("config", 0) for sh in shapes}):
        sel = [sh for sh in shapes if sh.get("config", 0) == cfg]
        us = sum(sh["us"] for sh in sel)
        roof = sum(sh["roof_us"] for sh in sel)
        flops = sum(sh["tflops"] * sh["us"] for sh in sel)   # TFLOPS x us = MFLOP
        gb = sum(sh["gbs"] * sh["us"] for sh in sel)
        e = dict(config=cfg, name=CONFIG_NAMES.get(cfg, "workload"), gemms=len(sel), us=us,
                 tflops=flops / us, gbs=gb / us, frac=roof / us,
                 bound=sorted({sh["bound"] for sh in sel}))
        if all("graph_us" in sh for sh in sel):
            g = sum(sh["graph_us"] for sh in sel)
            e.update(graph_us=g, graph_frac=roof / g if g > 0 else None)
        out.append(e)
    return out


def run_e2e(dg, dev, gemms, args, world):
    """Host buffers -> device, the GEMMs through the binding, outputs -> host, per step.  The
    copies run on their own streams, uploads on one and downloads on another (PCIe moves both
    directions at once), chained to the GEMMs by events: GEMM i waits for its inputs, the
    download of its output waits for GEMM i.  The step ends when the last output has landed in
    host memory, and every byte crosses PCIe inside the timed region."""
    host_in = [[t.cpu().pin_memory() for t in d.tensors_in()] for d in dev]
    host_out = [torch.empty(d.d.shape, dtype=d.d.dtype).pin_memory() for d in dev]
    h2d = sum(t.numel() * t.element_size() for ts in host_in for t in ts)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    n = len(dev)
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_out = [torch.cuda.Event() for _ in range(n)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def step():
        comp.synchronize()
        e0.record(up)
        with torch.cuda.stream(up):
            for i, (d, hs) in enumerate(zip(dev, host_in)):
                for dst, src in zip(d.tensors_in(), hs):
                    dst.copy_(src, non_blocking=True)
                ev_in[i].record(up)
        for i, d in enumerate(dev):
            comp.wait_event(ev_in[i])
            d.launch(comp)
            ev_out[i].record(comp)
        with torch.cuda.stream(down):
            for i, (d, ho) in enumerate(zip(dev, host_out)):
                down.wait_event(ev_out[i])
                ho.copy_(d.d, non_blocking=True)
            e1.record(down)
        e1.synchronize()
        return e0.elapsed_time(e1) * 1e-3

    for _ in range(min(args.warmup, 3)):
        step()
    steps = max(1, min(args.steps, 10))
    ts = [step() for _ in range(steps)]
    torch.cuda.synchronize()
    t_max = max_over_ranks(sum(ts), world, "cuda")
    flops = sum(g.flops for g in gemms)
    return dict(value=aggregate_tflops(flops, steps, world, t_max), unit=UNIT,
                h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h, steps=steps,
                ms_per_step=t_max / steps * 1e3,
                overlap="uploads, GEMMs and downloads on three streams chained by events")


# ---- CPU oracle (baseline and reference arm) --------------------------------------------------

def _oracle_rows(g: Gemm, rows_per_gemm: int, rng):
    import oracle
    c = g.case
    if g.kind == "dense":
        r = np.sort(rng.choice(c.M, size=min(c.M, rows_per_gemm), replace=False))
        oracle.gemm_dense(c.a, c.sa, g.oracle_b(), c.sb, rows=r)
        return 2.0 * len(r) * c.N * c.K
    if g.kind == "contiguous":
        valid = np.nonzero(c.m_indices >= 0)[0]
        r = np.sort(rng.choice(valid, size=min(len(valid), rows_per_gemm), replace=False))
        oracle.gemm_contiguous(c.a, c.sa, g.oracle_b(), c.sb, c.m_indices, rows=r)
        return 2.0 * len(r) * c.N * c.K
    flat = np.array([gi * c.M_max + r for gi in range(c.G) for r in range(int(c.masked_m[gi]))])
    r = np.sort(rng.choice(flat, size=min(len(flat), rows_per_gemm), replace=False))
    oracle.gemm_masked(c.a, c.sa, g.oracle_b(), c.sb, c.masked_m, rows=r)
    return 2.0 * len(r) * c.N * c.K


def oracle_sample_step(gemms, rows_per_gemm: int, rng) -> float:
    return sum(_oracle_rows(g, rows_per_gemm, rng) for g in gemms)


def cpu_baseline(gemms, budget_s: float = 15.0):
    """The oracle as it stands, on this host's cores, over seeded random rows of every GEMM of
    the step, repeated until about `budget_s` seconds of CPU work."""
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    rows = max(16, cores)
    rng = np.random.default_rng(1234)
    for g in gemms:
        g.oracle_b()  # an FP4 B is expanded once, outside the timed sample
    flops, t0, passes = 0.0, time.perf_counter(), 0
    while True:
        flops += oracle_sample_step(gemms, rows, rng)
        passes += 1
        if time.perf_counter() - t0 >= budget_s or passes >= 50:
            break
    dt = time.perf_counter() - t0
    return dict(value=flops / dt / 1e12, unit=UNIT, cores=cores, kind="oracle",
                sample=f"{passes} pass(es) of {rows} seeded random rows of every GEMM of the step "
                       f"({flops / 1e9:.1f} GFLOP in {dt:.1f} s, fp64, {cores} threads)")


def run_reference(args):
    """The CPU oracle on a bounded sample of the workload (rank 0 only)."""
    import oracle
    oracle.build()
    if args.workload in ("quant", "swiglu"):
        swiglu = args.workload == "swiglu"
        M, K = args.shape[:2] if args.shape else ((16384, 2048) if swiglu else (8192, 7168))
        rows = min(M, 256)
        bits = quant_input(M, 2 * K if swiglu else K)[:rows]
        fn = oracle.swiglu_quantize if swiglu else oracle.quantize_1x128
        for _ in range(args.warmup):
            fn(bits)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            fn(bits)
        dt = time.perf_counter() - t0
        value = args.steps * (swiglu_bytes(rows, K) if swiglu else quant_bytes(rows, K)) / dt / 1e9
        sample = f"the first {rows} rows per step"
        wl = (f"SwiGLU + per-token FP8 quantisation M={M} I={K}" if swiglu
              else f"per-token FP8 quantisation M={M} K={K}")
        return dict(metric=SWIGLU_METRIC if swiglu else QUANT_METRIC, value=value, unit="GB/s",
                    n_gpus=1, steps=args.steps,
                    warmup=args.warmup, ms_per_step=dt / args.steps * 1e3, higher_is_better=True,
                    scaling="weak", vs_baseline=None, dtype="f32", data="synthetic",
                    config=dict(workload=wl), impl="reference",
                    cpu_baseline=dict(value=value, unit="GB/s", cores=1, kind="oracle", sample=sample),
                    e2e=dict(value=value, unit="GB/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    gemms, desc = build_workload(args.workload, args.shape, args.fp4)
    for g in gemms:
        g.oracle_b()
    cores = os.cpu_count() or 1
    rows = 16
    rng = np.random.default_rng(99)
    for _ in range(args.warmup):
        oracle_sample_step(gemms, rows, rng)
    t0 = time.perf_counter()
    flops = 0.0
    for _ in range(args.steps):
        flops += oracle_sample_step(gemms, rows, rng)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    sample = f"{rows} seeded random rows of every GEMM of the step per step"
    return dict(metric=METRIC, value=value, unit=UNIT, n_gpus=1, steps=args.steps,
                warmup=args.warmup, ms_per_step=dt / args.steps * 1e3, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                config=bench_config(desc, len(gemms), 1), impl="reference",
                cpu_baseline=dict(value=value, unit=UNIT, cores=cores, kind="oracle", sample=sample),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))


# ---- the per-token FP8 quantisation (the step before the GEMM) ----------------------------------

QUANT_METRIC = ("GB/s of the per-token FP8 quantisation (bf16 -> e4m3 codes + fp32 1x128 scales) "
                "at 1 B200; fraction of the HBM roofline")


def quant_input(M: int, K: int, seed: int = 7000) -> np.ndarray:
    """bf16 bits [M][K]: N(0,1) activations with 1 % outliers x50 (seeded, CPU)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g)
    mask = torch.rand(M, K, generator=g) < 0.01
    x = torch.where(mask, x * 50.0, x)
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def quant_bytes(M: int, K: int) -> float:
    return 2.0 * M * K + M * K + 4.0 * M * (K // 128)


SWIGLU_METRIC = ("GB/s of SwiGLU + per-token FP8 quantisation (bf16 gate|up [M, 2I] -> e4m3 [M, I] + "
                 "fp32 1x128 scales) at 1 B200; fraction of the HBM roofline")


def swiglu_bytes(M: int, I: int) -> float:
    return 2.0 * M * 2 * I + M * I + 4.0 * M * (I // 128)


def run_quant(args, rank, world, local_rank):
    """--workload quant: the per-token quantisation of an M x K activation (default 8192 x 7168);
    --workload swiglu: SwiGLU + quantisation of an M x 2I gate|up tensor (default 16384 x 2*2048,
    the per-expert intermediate width of DeepSeek-V3's MoE)."""
    import fp8_block_scaled_tma_b200 as dg
    torch.cuda.set_device(local_rank)
    swiglu = args.workload == "swiglu"
    if swiglu:
        M, K = args.shape[:2] if args.shape else (16384, 2048)  # K = I
        bits = quant_input(M, 2 * K)
    else:
        M, K = args.shape[:2] if args.shape else (8192, 7168)
        bits = quant_input(M, K)
    x = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    q = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    sfa = torch.empty(K // 128, dg.get_tma_aligned_size(M, 4), dtype=torch.float32, device="cuda")

    def run_kernel():
        if swiglu:
            dg.swiglu_quantize_fp8_1x128(x, None, 0, q, sfa)
        else:
            dg.quantize_fp8_1x128(x, q, sfa)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def step():
        torch.cuda._sleep(200_000)
        flush.fill_(1)
        e0.record(stream)
        run_kernel()
        e1.record(stream)
        stream.synchronize()
        return e0.elapsed_time(e1) * 1e-3

    for _ in range(args.warmup):
        step()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        ts = [step() for _ in range(args.steps)]
    torch.cuda.synchronize()
    if dg.poll_device_error(stream) != 0:
        raise RuntimeError("device error")
    total = max_over_ranks(sum(ts), world, "cuda")
    nbytes = swiglu_bytes(M, K) if swiglu else quant_bytes(M, K)
    value = world * nbytes * args.steps / total / 1e9
    peaks = load_peaks()
    per = statistics.mean(ts)
    achieved = nbytes / per / 1e9
    roof = dict(bound="hbm", achieved=achieved, peak=peaks["hbm_gbs"], unit="GB/s",
                frac=achieved / peaks["hbm_gbs"], frac_spec=achieved / SPEC_HBM_GBS,
                peak_source=f"{peaks['source']} HBM copy",
                kernel=(f"dg_swiglu_quantize_1x128_kernel {M}x{2 * K}" if swiglu
                        else f"dg_quantize_1x128_kernel {M}x{K}"),
                traffic_unit="bytes/launch")
    roof["traffic"], roof["traffic_source"] = measured_traffic(roof["kernel"], args.traffic_bytes)
    # e2e: pinned host bf16 in, quantise, codes and scales out
    hx = x.cpu().pin_memory()
    hq = torch.empty_like(q, device="cpu").pin_memory()
    hs = torch.empty_like(sfa, device="cpu").pin_memory()

    def e2e_step():
        e0.record(stream)
        x.copy_(hx, non_blocking=True)
        run_kernel()
        hq.copy_(q, non_blocking=True)
        hs.copy_(sfa, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) * 1e-3

    e2e_step()
    et = [e2e_step() for _ in range(5)]
    e2e_t = max_over_ranks(sum(et), world, "cuda")
    out = dict(metric=SWIGLU_METRIC if swiglu else QUANT_METRIC, value=value, unit="GB/s",
               n_gpus=world, steps=args.steps,
               warmup=args.warmup, ms_per_step=total / args.steps * 1e3, higher_is_better=True,
               scaling="weak", vs_baseline=None, dtype="bf16 -> e4m3 (fp32 arithmetic)",
               data="synthetic",
               config=dict(workload=(f"SwiGLU + per-token FP8 quantisation M={M} I={K}" if swiglu
                                     else f"per-token FP8 quantisation M={M} K={K}")
                                    + ", N(0,1) with 1% x50 outliers",
                           l2=f"256 MiB write before every launch; input + output {nbytes / 1e6:.0f} MB > L2"),
               roofline=roof, gpu_launches=args.steps, clocks=clk.summary(),
               e2e=dict(value=world * nbytes * 5 / e2e_t / 1e9, unit="GB/s",
                        h2d_bytes_per_step=hx.numel() * 2, d2h_bytes_per_step=hq.numel() + hs.numel() * 4))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        rows = min(M, 512)
        t0 = time.perf_counter()
        passes = 0
        while time.perf_counter() - t0 < min(args.cpu_seconds, 5.0):
            if swiglu:
                oracle.swiglu_quantize(bits[:rows])
            else:
                oracle.quantize_1x128(bits[:rows])
            passes += 1
        dt = time.perf_counter() - t0
        per_pass = swiglu_bytes(rows, K) if swiglu else quant_bytes(rows, K)
        out["cpu_baseline"] = dict(value=passes * per_pass / dt / 1e9, unit="GB/s", cores=1,
                                   kind="oracle", sample=f"{passes} pass(es) over the first {rows} rows")
    return out


# ---- main ---------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["sweep", "small", "contiguous", "masked", "prefill",
                                           "dense", "quant", "swiglu", "all"], default="all")
    ap.add_argument("--shape", type=lambda v: tuple(int(x) for x in v.split(",")), default=None,
                    help="M,N,K of --workload dense; M,K of --workload quant; M,I of --workload swiglu")
    ap.add_argument("--block-n", type=int, default=0, help="tile override (tuning)")
    ap.add_argument("--stages", type=int, default=0, help="pipeline-stage override (tuning)")
    ap.add_argument("--splits", type=int, default=0, help="split-K override (tuning)")
    ap.add_argument("--family", type=int, default=0,
                    help="kernel family override (tuning): 1 one-CTA, 2 CTA pair, 3 split-K")
    ap.add_argument("--fp4", action="store_true",
                    help="B of every GEMM as packed FP4 E2M1 (the FP8 x FP4 entries)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph timing of memory-bound shapes")
    ap.add_argument("--no-cublas", action="store_true", help="skip the cuBLAS FP8 measuring stick")
    ap.add_argument("--no-library-stick", action="store_true",
                    help="skip the block-scaled FP8 library measuring stick")
    ap.add_argument("--library-stick", default=None, help=argparse.SUPPRESS)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel from an ncu capture")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.fp4 and args.workload in ("quant", "swiglu"):
        raise SystemExit("--fp4 applies to the GEMM workloads")
    if args.workload == "dense" and (args.shape is None or len(args.shape) != 3):
        raise SystemExit("--workload dense needs --shape M,N,K")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.library_stick:
        print(json.dumps(run_library_stick(args.library_stick, args.steps)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        out = (run_quant if args.workload in ("quant", "swiglu") else run_ours)(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
