"""Parity helpers shared by the GPU tests: moving seeded inputs to the device, running the
library, and comparing with the oracle under the stated tolerance.

Tolerance (per element, on valid rows):  |D - Dref| <= 2 * ulp_bf16(Dref) + 1e-3 * sum_k |sa a| |sb b|
with ulp_bf16(x) = 2^(max(floor(log2 |x|), -126) - 7) (2^-133 for x = 0); and per matrix
1 - 2<D,Dref> / (<D,D> + <Dref,Dref>) <= 1e-5 in fp64.  Rows the call must not write keep the
sentinel bit pattern exactly.

Every comparison also bounds the error beyond the final bf16 rounding ("excess", see
``compare``) by 1e-5 of sum_k |sa a| |sb b|.  That is what fp32 accumulation of the 128-wide
K-slice partials allows (one fp32 rounding per slice and per promotion: at most about
(K/128 + 1) * 2^-24 relative to the magnitude, 8.6e-6 at K = 18432), and what an accumulator
of fewer bits -- the FP8 tensor-core imprecision that two-level accumulation exists to contain
(DeepGEMM release write-up, "深入了解DeepGEMM") -- would exceed.
"""
from __future__ import annotations

import numpy as np
import torch

SENTINEL = 0xFFFF  # a bf16 NaN pattern no finite result can take
ULP_FACTOR = 2.0
MAG_FACTOR = 1e-3
DIFF_MAX = 1e-5
EXCESS_MAX = 1e-5


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def ulp_bf16(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.where(ax > 0, np.maximum(e, -126), -126)
    return np.exp2(e - 7)


def compare(got_bits: np.ndarray, ref_bits: np.ndarray, mag: np.ndarray, acc=None) -> dict:
    """Element and matrix checks over matching arrays of valid entries.  With ``acc`` (the
    oracle's fp64 value before rounding) it also reports the error beyond one bf16 rounding:
    excess = max(0, |D - acc| - ulp_bf16(acc)) / mag, which fp32 accumulation keeps near 1e-6."""
    got = bits_to_f64(got_bits)
    ref = bits_to_f64(ref_bits)
    assert np.all(np.isfinite(ref)), "oracle produced a non-finite value"
    err = np.abs(got - ref)
    bound = ULP_FACTOR * ulp_bf16(ref) + MAG_FACTOR * mag
    bad = ~(err <= bound)
    den = float(np.sum(got * got) + np.sum(ref * ref))
    diff = 0.0 if den == 0 else 1.0 - 2.0 * float(np.sum(got * ref)) / den
    excess = 0.0
    if acc is not None and err.size:
        acc = np.asarray(acc, dtype=np.float64)
        ex = np.maximum(0.0, np.abs(got - acc) - ulp_bf16(acc)) / np.maximum(mag, 1e-300)
        excess = float(np.max(ex))
    return dict(n_bad=int(bad.sum()), n=int(err.size), diff=diff, excess=excess,
                first_bad=None if not bad.any() else tuple(int(i) for i in np.argwhere(bad)[0]))


def assert_close(got_bits, ref_bits, mag, what: str, acc, matrix: bool = True) -> dict:
    """The parity bar: every element within tolerance, the matrix difference within DIFF_MAX,
    and the error beyond one bf16 rounding within EXCESS_MAX of the magnitude.  ``acc`` is the
    oracle's unrounded fp64 result for the same entries (required).

    matrix=False drops the matrix criterion, for inputs built so that every exact result is the
    residue of a catastrophic cancellation (|Dref| ~ 1e-8 of sum |ab|).  There the matrix
    difference compares errors of fp32 accumulation (~2^-24 of the cancelled magnitude, which
    the two-level method accepts inside each 128-wide slice) with the tiny residues themselves,
    and no fp32-accumulating implementation meets it; the element and excess bounds, which are
    relative to the magnitude, still apply."""
    r = compare(got_bits, ref_bits, mag, acc)
    assert r["n_bad"] == 0, f"{what}: {r['n_bad']}/{r['n']} elements out of tolerance, first at {r['first_bad']}: {r}"
    if matrix:
        assert r["diff"] <= DIFF_MAX, f"{what}: matrix diff {r['diff']} > {DIFF_MAX}"
    assert r["excess"] < EXCESS_MAX, f"{what}: error beyond one bf16 rounding {r['excess']} >= {EXCESS_MAX}"
    return r


def check(got_bits, ref, what: str, sel=None, matrix: bool = True) -> dict:
    """assert_close against an oracle Result, optionally on a selection ``sel`` (an index or
    mask applied alike to the GPU bits and to the oracle's arrays)."""
    if sel is None:
        return assert_close(got_bits, ref.bits, ref.mag, what, ref.acc, matrix)
    return assert_close(got_bits[sel], ref.bits[sel], ref.mag[sel], what, ref.acc[sel], matrix)


def to_dev_u8(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def to_dev_f32(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def sentinel_out(shape) -> torch.Tensor:
    # int16 -1 is the bit pattern 0xFFFF (SENTINEL)
    return torch.full(shape, -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)


def out_bits(d: torch.Tensor) -> np.ndarray:
    return d.view(torch.int16).cpu().numpy().view(np.uint16)


def run_dense(dg, case, d=None, workspace=None) -> torch.Tensor:
    a = to_dev_u8(case.a)
    b = to_dev_u8(case.b)
    sfa = dg.sfa_mn_major(to_dev_f32(case.sa))
    sfb = to_dev_f32(case.sb)
    if d is None:
        d = sentinel_out((case.M, case.N))
    dg.dg_gemm_fp8_fp8_bf16_nt(a, sfa, b, sfb, d, workspace=workspace)
    torch.cuda.synchronize()
    return d


def run_contiguous(dg, case, a=None, sa=None) -> torch.Tensor:
    a = to_dev_u8(case.a if a is None else a)
    sfa = dg.sfa_mn_major(to_dev_f32(case.sa if sa is None else sa))
    b = to_dev_u8(case.b)
    sfb = to_dev_f32(case.sb)
    mi = torch.from_numpy(case.m_indices).cuda()
    d = sentinel_out((case.M_total, case.N))
    dg.dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(a, sfa, b, sfb, d, mi)
    torch.cuda.synchronize()
    return d


def run_masked(dg, case, a=None, sa=None) -> torch.Tensor:
    a = to_dev_u8(case.a if a is None else a)
    sfa = dg.sfa_mn_major(to_dev_f32(case.sa if sa is None else sa))
    b = to_dev_u8(case.b)
    sfb = to_dev_f32(case.sb)
    mm = torch.from_numpy(case.masked_m).cuda()
    d = sentinel_out((case.G, case.M_max, case.N))
    dg.dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(a, sfa, b, sfb, d, mm, case.expected_m)
    torch.cuda.synchronize()
    return d


def run_dense_fp4(dg, case, d=None) -> torch.Tensor:
    """case.b holds packed E2M1 bytes [N, K/2]."""
    a = to_dev_u8(case.a)
    b = to_dev_u8(case.b)
    sfa = dg.sfa_mn_major(to_dev_f32(case.sa))
    sfb = to_dev_f32(case.sb)
    if d is None:
        d = sentinel_out((case.M, case.N))
    dg.dg_gemm_fp8_fp4_bf16_nt(a, sfa, b, sfb, d)
    torch.cuda.synchronize()
    return d


def run_contiguous_fp4(dg, case) -> torch.Tensor:
    a = to_dev_u8(case.a)
    sfa = dg.sfa_mn_major(to_dev_f32(case.sa))
    b = to_dev_u8(case.b)
    sfb = to_dev_f32(case.sb)
    mi = torch.from_numpy(case.m_indices).cuda()
    d = sentinel_out((case.M_total, case.N))
    dg.dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous(a, sfa, b, sfb, d, mi)
    torch.cuda.synchronize()
    return d


def run_masked_fp4(dg, case) -> torch.Tensor:
    a = to_dev_u8(case.a)
    sfa = dg.sfa_mn_major(to_dev_f32(case.sa))
    b = to_dev_u8(case.b)
    sfb = to_dev_f32(case.sb)
    mm = torch.from_numpy(case.masked_m).cuda()
    d = sentinel_out((case.G, case.M_max, case.N))
    dg.dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked(a, sfa, b, sfb, d, mm, case.expected_m)
    torch.cuda.synchronize()
    return d


def sample_rows(M: int, n: int, seed: int) -> np.ndarray:
    """Rows at tile boundaries (first/last rows of the first, second and last 128-row tiles),
    one seeded row in EVERY 128-row tile (so that a tile written to the wrong place, or not
    at all, cannot hide between samples), plus n seeded random rows."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 129, 255, M - 129, M - 128, M - 2, M - 1]
    rows = set(r for r in fixed if 0 <= r < M)
    for t0 in range(0, M, 128):
        rows.add(int(rng.integers(t0, min(t0 + 128, M))))
    rows.update(int(r) for r in rng.integers(0, M, size=min(n, M)))
    return np.array(sorted(rows), dtype=np.int64)


def sample_valid_rows(valid: np.ndarray, n: int, seed: int) -> np.ndarray:
    """For a grouped layout with a per-row validity mask: the first and last valid rows, one
    seeded valid row in every 128-row tile that has one, plus n seeded valid rows."""
    rng = np.random.default_rng(seed)
    idx = np.nonzero(valid)[0]
    rows = set(int(r) for r in idx[:2]) | set(int(r) for r in idx[-2:])
    for t0 in range(0, len(valid), 128):
        v = idx[(idx >= t0) & (idx < t0 + 128)]
        if v.size:
            rows.add(int(rng.choice(v)))
    if idx.size:
        rows.update(int(r) for r in rng.choice(idx, size=min(n, idx.size), replace=False))
    return np.array(sorted(rows), dtype=np.int64)
