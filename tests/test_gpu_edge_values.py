"""GPU parity on the values two-level accumulation exists for (DeepGEMM release write-up,
"深入了解DeepGEMM": the FP8 tensor cores accumulate imprecisely, so each 128-wide K slice is
promoted into an fp32 accumulator on the CUDA cores).  Every kernel family -- one-CTA, CTA pair,
split-K cluster, swapped operands -- plus one contiguous segment and one masked group, with B
as E4M3 and as packed E2M1, meets inputs whose codes are drawn directly (``workloads.edge_*``):

  cancel           the two largest products of every slice (+-448 x +-448) cancel exactly and
                   the rest are products of subnormal codes;
  cancel_residual  the same, leaving a residual next to the tiny products;
  pm_max           every code +-448 (E2M1 +-6): slice sums up to 128 * 448^2 > 2^24;
  all_codes        codes uniform over all 254 finite E4M3 codes (all 16 E2M1 codes);

with power-of-two block scales whose products span 2^-60 .. 2^60.  Each result is compared with
the oracle under the parity tolerance, the matrix bound, and the bound on the error beyond one
bf16 rounding (1e-5 of sum |sa a| |sb b|).

``test_in_slice_accumulation_probe`` measures what the tensor core does inside one slice: the
two cancelling products sit in the same 32-wide MMA step or in different ones, and the result
(sa = sb = 1, K = 128) is compared with the exact sum of the tiny products.  With
DG_EDGE_REPORT=<path> the largest excess per family and the probe's figures are written there.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu

N_EDGE, K_EDGE = 320, 1024          # a ragged last 64-column scale block, 8 K blocks
PATHS = {
    # name: (layout, kernel family, rows)
    "one-CTA": ("dense", 1, 264),
    "CTA pair": ("dense", 2, 264),
    "split-K": ("dense", 3, 200),
    "swapped": ("dense", 4, 100),
    "contiguous": ("contiguous", 1, 200),
    "masked one-CTA": ("masked", 1, 200),
    "masked pair": ("masked", 2, 200),
}
_REPORT: dict = {"excess": {}, "probe": {}}


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fp8_block_scaled_tma_b200 as mod
    mod.set_config_override(0, 0)
    mod.set_num_sms(0)
    mod.set_kernel_family(0)
    assert mod.poll_device_error() == 0
    yield mod
    mod.set_config_override(0, 0)
    mod.set_kernel_family(0)
    path = os.environ.get("DG_EDGE_REPORT")
    if path:
        with open(path, "w") as f:
            json.dump(_REPORT, f, indent=1, sort_keys=True)


@pytest.fixture(scope="module")
def orc():
    import oracle
    oracle.build()
    return oracle


def _run(dg, orc, path, pattern, fp4, seed):
    layout, family, rows = PATHS[path]
    dg.set_kernel_family(family)
    try:
        if layout == "dense":
            case = workloads.edge_dense(pattern, rows, N_EDGE, K_EDGE, seed, fp4=fp4)
            got = P.out_bits(P.run_dense_fp4(dg, case) if fp4 else P.run_dense(dg, case))
            used = dg.get_last_launch()["family"]
            b = orc.e2m1_to_e4m3(case.b) if fp4 else case.b
            ref = orc.gemm_dense(case.a, case.sa, b, case.sb)
            sel = None
            assert not np.any(got == P.SENTINEL)
        elif layout == "contiguous":
            case = workloads.edge_contiguous(pattern, N_EDGE, K_EDGE, seed, rows=rows, fp4=fp4)
            got = P.out_bits(P.run_contiguous_fp4(dg, case) if fp4 else P.run_contiguous(dg, case))
            used = dg.get_last_launch()["family"]
            b = orc.e2m1_to_e4m3(case.b) if fp4 else case.b
            ref = orc.gemm_contiguous(case.a, case.sa, b, case.sb, case.m_indices)
            sel = case.m_indices >= 0
            assert np.all(got[~sel] == P.SENTINEL), "a padding row was written"
        else:
            case = workloads.edge_masked(pattern, N_EDGE, K_EDGE, seed, rows=rows, fp4=fp4)
            got = P.out_bits(P.run_masked_fp4(dg, case) if fp4 else P.run_masked(dg, case))
            used = dg.get_last_launch()["family"]
            b = orc.e2m1_to_e4m3(case.b) if fp4 else case.b
            ref = orc.gemm_masked(case.a, case.sa, b, case.sb, case.masked_m)
            sel = np.arange(case.M_max)[None, :] < case.masked_m[:, None]
            assert np.all(got[~sel] == P.SENTINEL), "a row beyond masked_m was written"
    finally:
        dg.set_kernel_family(0)
    assert used == family, f"{path}: ran kernel family {used}, not {family}"
    # the pure cancellation inputs: element and excess bounds (relative to the magnitude);
    # the matrix criterion is recorded, not asserted (see parity.assert_close)
    r = P.check(got, ref, f"{path} {pattern}{' fp4' if fp4 else ''}", sel=sel,
                matrix=pattern != "cancel")
    assert dg.poll_device_error() == 0
    key = f"{path}{' fp4' if fp4 else ''}"
    _REPORT["excess"][key] = max(_REPORT["excess"].get(key, 0.0), r["excess"])
    same = got == ref.bits if sel is None else got[sel] == ref.bits[sel]
    k2 = f"{key} {pattern}"
    _REPORT.setdefault("bit_exact_fraction", {})[k2] = float(np.mean(same))
    _REPORT.setdefault("matrix_diff", {})[k2] = r["diff"]
    return r


@pytest.mark.parametrize("pattern", workloads.EDGE_PATTERNS)
@pytest.mark.parametrize("path", list(PATHS))
def test_edge_values_fp8(dg, orc, path, pattern):
    _run(dg, orc, path, pattern, False, seed=101 + workloads.EDGE_PATTERNS.index(pattern))


@pytest.mark.parametrize("pattern", workloads.EDGE_PATTERNS)
@pytest.mark.parametrize("path", list(PATHS))
def test_edge_values_fp4(dg, orc, path, pattern):
    _run(dg, orc, path, pattern, True, seed=201 + workloads.EDGE_PATTERNS.index(pattern))


def test_edge_scale_extremes_reach_the_range(dg, orc):
    """The power-of-two scales really reach 2^+-60 in their products, and the results keep
    their dynamic range (no flush to zero or overflow on the way)."""
    case = workloads.edge_dense("pm_max", 264, N_EDGE, K_EDGE, seed=7)
    prod = np.log2(case.sa[:, None, :]) + np.log2(case.sb[None, :, :])
    assert prod.min() <= -55 and prod.max() >= 55
    got = P.out_bits(P.run_dense(dg, case))
    ref = orc.gemm_dense(case.a, case.sa, case.b, case.sb)
    P.check(got, ref, "scale extremes")
    v = np.abs(P.bits_to_f64(got))
    assert v.max() > 2.0 ** 75 and v[v > 0].min() < 1.0


def _probe_case(M, N, same_step: bool, seed: int):
    """One K block (K = 128), unit scales.  A row m: +-448 at k0 and k1 (the same sign), small
    codes elsewhere; B row n: +-448 at k0 and the opposite sign at k1.  k0 and k1 lie in the
    same 32-wide MMA step (same_step) or in different steps."""
    rng = np.random.default_rng(seed)
    K = 128
    if same_step:
        s = int(rng.integers(0, 4))
        k0, k1 = (32 * s + rng.choice(32, 2, replace=False)).tolist()
    else:
        s0, s1 = rng.choice(4, 2, replace=False)
        k0, k1 = int(32 * s0 + rng.integers(0, 32)), int(32 * s1 + rng.integers(0, 32))
    small = lambda r: (rng.integers(1, 13, (r, K)) | (rng.integers(0, 2, (r, K)) << 7)).astype(np.uint8)
    a, b = small(M), small(N)
    sgn_a = rng.integers(0, 2, M).astype(np.uint8) << 7
    sgn_b = rng.integers(0, 2, N).astype(np.uint8) << 7
    a[:, k0] = 0x7E | sgn_a
    a[:, k1] = 0x7E | sgn_a
    b[:, k0] = 0x7E | sgn_b
    b[:, k1] = 0x7E | (sgn_b ^ 0x80)
    sa = np.ones((M, 1), np.float32)
    sb = np.ones((-(-N // 128), 1), np.float32)
    return workloads.Dense(M, N, K, a, sa, b, sb), (k0, k1)


@pytest.mark.parametrize("same_step", [True, False])
def test_in_slice_accumulation_probe(dg, orc, same_step):
    """Measures the tensor core's accumulation inside one slice where two +-448^2 products
    cancel: the exact result is the sum of the tiny products.  Asserts the parity bar and
    records how far the GPU result sits from the exact one, in bf16 ulps of the exact value
    and relative to 448^2 (the size of the cancelled terms)."""
    worst_ulps, worst_rel, exact_frac, diffs = 0.0, 0.0, [], []
    for seed in range(8):
        case, _ = _probe_case(128, 256, same_step, seed=900 + seed + (100 if same_step else 0))
        for family in (1, 4):
            dg.set_kernel_family(family)
            try:
                got = P.out_bits(P.run_dense(dg, case))
            finally:
                dg.set_kernel_family(0)
            ref = orc.gemm_dense(case.a, case.sa, case.b, case.sb)
            r = P.check(got, ref, f"probe family {family}", matrix=False)
            diffs.append(r["diff"])
            g = P.bits_to_f64(got)
            err = np.abs(g - ref.acc)
            nz = ref.acc != 0
            worst_ulps = max(worst_ulps, float(np.max(err[nz] / P.ulp_bf16(ref.acc[nz]))))
            worst_rel = max(worst_rel, float(np.max(err)) / 448.0 ** 2)
            exact_frac.append(float(np.mean(got == ref.bits)))
    _REPORT["probe"]["same MMA step" if same_step else "different MMA steps"] = dict(
        max_err_bf16_ulps_of_exact=worst_ulps, max_err_over_448sq=worst_rel,
        min_fraction_bit_exact=min(exact_frac), max_matrix_diff=max(diffs))
    assert dg.poll_device_error() == 0
