"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on the same seeded
inputs, element by element, for the dense, contiguous-grouped and masked-grouped GEMMs.
Small cases are compared in full; full-size workloads on sampled rows (boundary rows of the
first and last tiles plus seeded random rows), with untouched rows checked in full."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fp8_block_scaled_tma_b200 as mod
    mod.set_config_override(0, 0)
    mod.set_num_sms(0)
    assert mod.poll_device_error() == 0
    yield mod
    mod.set_config_override(0, 0)
    mod.set_num_sms(0)


@pytest.fixture(scope="module")
def orc():
    import oracle
    oracle.build()
    return oracle


def _dense_full_check(dg, orc, case, what):
    d = P.run_dense(dg, case)
    got = P.out_bits(d)
    ref = orc.gemm_dense(case.a, case.sa, case.b, case.sb)
    r = P.assert_close(got, ref.bits, ref.mag, what, acc=ref.acc)
    assert dg.poll_device_error() == 0
    return r


def test_small_dense_config(dg, orc):
    """128 x 256 x 512, A and B ~ N(0, 1): compared in full."""
    _dense_full_check(dg, orc, workloads.small_dense(), "small dense")


@pytest.mark.parametrize("M,N,K", [
    (1, 8, 128), (1, 2112, 256), (7, 136, 384), (130, 264, 256), (200, 2112, 1024),
    (257, 520, 384), (384, 1024, 1536), (64, 4096, 512), (1000, 96, 128),
])
def test_dense_ragged_shapes(dg, orc, M, N, K):
    case = workloads.dense(M, N, K, seed=M * 7 + N * 3 + K, a_std=1.0, b_std=0.02)
    _dense_full_check(dg, orc, case, f"dense {M}x{N}x{K}")


@pytest.mark.parametrize("bn", [32, 64, 96, 128, 160, 192, 224, 256])
def test_dense_every_block_n(dg, orc, bn):
    case = workloads.dense(300, 1000, 640, seed=bn)
    dg.set_config_override(bn, 0)
    try:
        r = _dense_full_check(dg, orc, case, f"BN={bn}")
        assert dg.get_last_launch()["block_n"] == bn
    finally:
        dg.set_config_override(0, 0)
    # beyond the final bf16 rounding, only fp32 accumulation error remains
    assert r["excess"] < 1e-5, r


@pytest.mark.parametrize("stages", [2, 3])
def test_dense_few_stages(dg, orc, stages):
    case = workloads.dense(256, 512, 2048, seed=77)
    dg.set_config_override(128, stages)
    try:
        _dense_full_check(dg, orc, case, f"stages={stages}")
        assert dg.get_last_launch()["stages"] == stages
    finally:
        dg.set_config_override(0, 0)


def test_dense_sm_cap_many_tiles_per_cta(dg, orc):
    """7 CTAs walk 40 tiles each: exercises the persistent loop and the stage/phase wrap."""
    case = workloads.dense(1024, 2560, 512, seed=91)
    prev = dg.set_num_sms(7)
    try:
        dg.set_config_override(64, 0)
        _dense_full_check(dg, orc, case, "sm cap 7")
        assert dg.get_last_launch()["grid"] == 7
    finally:
        dg.set_config_override(0, 0)
        dg.set_num_sms(prev)


def test_dense_deterministic(dg):
    case = workloads.dense(512, 2112, 1024, seed=5)
    a = P.out_bits(P.run_dense(dg, case))
    b = P.out_bits(P.run_dense(dg, case))
    assert np.array_equal(a, b)


@pytest.mark.parametrize("i", range(15))
def test_dense_sweep_full_size_sampled(dg, orc, i):
    """The 15 shapes of the dense sweep at full size; all outputs written and finite, sampled
    rows against the oracle."""
    case = workloads.sweep_case(i)
    d = P.run_dense(dg, case)
    got = P.out_bits(d)
    assert not np.any(got == P.SENTINEL)
    assert np.all(np.isfinite(P.bits_to_f64(got)))
    rows = P.sample_rows(case.M, 24, seed=i)
    ref = orc.gemm_dense(case.a, case.sa, case.b, case.sb, rows=rows)
    P.check(got[rows], ref, f"sweep {i} {case.M}x{case.N}x{case.K}")


def test_prefill_full_size_sampled(dg, orc):
    """8192 x 7168 x 18432 with 1% x50 outliers in A."""
    case = workloads.prefill_case()
    d = P.run_dense(dg, case)
    got = P.out_bits(d)
    assert not np.any(got == P.SENTINEL)
    rows = P.sample_rows(case.M, 40, seed=55)
    ref = orc.gemm_dense(case.a, case.sa, case.b, case.sb, rows=rows)
    P.check(got[rows], ref, "prefill")


# ---- contiguous ----------------------------------------------------------------------------

def _contig_check(dg, orc, case, rows=None, what="contiguous"):
    d = P.run_contiguous(dg, case)
    got = P.out_bits(d)
    pad = case.m_indices < 0
    assert np.all(got[pad] == P.SENTINEL), "a padding row was written"
    ref = orc.gemm_contiguous(case.a, case.sa, case.b, case.sb, case.m_indices, rows=rows)
    check = ~pad if rows is None else np.isin(np.arange(case.M_total), rows) & ~pad
    P.check(got, ref, what, sel=check)
    assert dg.poll_device_error() == 0
    return got


def test_contiguous_small_full(dg, orc):
    case = workloads.contiguous(G=4, N=264, K=384, seed=12, counts=[5, 130, 0, 128])
    _contig_check(dg, orc, case)


def test_contiguous_all_padding_tile(dg, orc):
    """A whole 128-row tile of -1 rows between two experts is skipped and left untouched."""
    case = workloads.contiguous(G=2, N=128, K=256, seed=13, counts=[100, 60])
    mi = case.m_indices.copy()
    # insert an all-padding tile after expert 0's segment
    ins = np.full(128, -1, np.int32)
    case.m_indices = np.concatenate([mi[:128], ins, mi[128:]])
    case.a = np.concatenate([case.a[:128], case.a[:128], case.a[128:]])
    case.sa = np.concatenate([case.sa[:128], case.sa[:128], case.sa[128:]])
    _contig_check(dg, orc, case, what="all-padding tile")


def test_contiguous_config_full_size_sampled(dg, orc):
    case = workloads.contiguous_case()
    rows = P.sample_valid_rows(case.m_indices >= 0, 40, seed=3)
    _contig_check(dg, orc, case, rows=rows, what="contiguous config")


def test_contiguous_nan_in_padding_rows_isolated(dg, orc):
    """Padding rows of A hold NaN codes and NaN scales: the valid rows are unchanged."""
    case = workloads.contiguous(G=3, N=256, K=512, seed=14, counts=[70, 129, 1])
    clean = P.out_bits(P.run_contiguous(dg, case))
    a = case.a.copy()
    sa = case.sa.copy()
    pad = case.m_indices < 0
    a[pad] = 0x7F
    sa[pad] = np.nan
    dirty = P.out_bits(P.run_contiguous(dg, case, a=a, sa=sa))
    assert np.array_equal(clean[~pad], dirty[~pad])
    assert np.all(np.isfinite(P.bits_to_f64(dirty[~pad])))
    assert np.all(dirty[pad] == P.SENTINEL)


def test_contiguous_index_below_minus_one_reports_layout_error(dg, orc):
    """An expert index below -1 (only -1 marks padding) breaks the layout contract: the device
    sets DG_ERR_LAYOUT, the row is not written, and the other rows are still correct -- also
    when a whole tile holds such indices."""
    case = workloads.contiguous(G=2, N=128, K=256, seed=16, counts=[128, 100])
    case.m_indices = case.m_indices.copy()
    case.m_indices[5] = -2
    case.m_indices[200] = np.iinfo(np.int32).min
    got = P.out_bits(P.run_contiguous(dg, case))
    assert dg.poll_device_error() == dg.DG_ERR_LAYOUT
    assert np.all(got[5] == P.SENTINEL) and np.all(got[200] == P.SENTINEL)
    ok = case.m_indices >= 0
    ref = orc.gemm_contiguous(case.a, case.sa, case.b, case.sb, np.where(ok, case.m_indices, -1))
    P.check(got, ref, "index below -1", sel=ok)
    assert np.all(got[~ok] == P.SENTINEL)
    # a tile whose every index is -2 is skipped and still reported
    case2 = workloads.contiguous(G=1, N=64, K=128, seed=17, counts=[128])
    case2.m_indices = np.full_like(case2.m_indices, -2)
    got2 = P.out_bits(P.run_contiguous(dg, case2))
    assert dg.poll_device_error() == dg.DG_ERR_LAYOUT
    assert np.all(got2 == P.SENTINEL)


def test_contiguous_mixed_expert_tile_reports_layout_error(dg):
    """A 128-row tile whose rows name two experts breaks the layout contract: the device sets
    DG_ERR_LAYOUT and the rows of the other expert are not written."""
    case = workloads.contiguous(G=2, N=64, K=128, seed=15, counts=[128, 128])
    case.m_indices = case.m_indices.copy()
    case.m_indices[10] = 1
    got = P.out_bits(P.run_contiguous(dg, case))
    assert dg.poll_device_error() == dg.DG_ERR_LAYOUT
    assert np.all(got[10] == P.SENTINEL)
    assert not np.any(got[11:128] == P.SENTINEL)


# ---- masked --------------------------------------------------------------------------------

def _masked_check(dg, orc, case, rows=None, what="masked"):
    d = P.run_masked(dg, case)
    got = P.out_bits(d)
    r_idx = np.arange(case.M_max)[None, :]
    invalid = r_idx >= case.masked_m[:, None]
    assert np.all(got[invalid] == P.SENTINEL), "a row beyond masked_m was written"
    ref = orc.gemm_masked(case.a, case.sa, case.b, case.sb, case.masked_m, rows=rows)
    valid = ~invalid
    if rows is not None:
        sel = np.zeros(case.G * case.M_max, bool)
        sel[rows] = True
        valid &= sel.reshape(case.G, case.M_max)
    P.check(got, ref, what, sel=valid)
    assert dg.poll_device_error() == 0
    return got


def test_masked_small_edge_counts(dg, orc):
    case = workloads.masked(G=6, M_max=256, N=136, K=256, seed=21,
                            masked_m=[0, 1, 127, 128, 129, 256])
    _masked_check(dg, orc, case)


def test_masked_all_empty(dg, orc):
    case = workloads.masked(G=3, M_max=128, N=64, K=128, seed=22, masked_m=[0, 0, 0])
    _masked_check(dg, orc, case)


@pytest.mark.parametrize("family", [1, 2])
def test_masked_largest_group_count(dg, orc, family):
    """G = 1024, the largest group count the masked call takes: the tile prefix over groups
    fills its last slot.  Most groups are empty; the last group and a few others hold rows."""
    G = 1024
    mm = np.zeros(G, np.int64)
    mm[[0, 3, 511, 1000, G - 1]] = [128, 1, 77, 128, 100]
    case = workloads.masked(G=G, M_max=128, N=256, K=128, seed=26, masked_m=mm)
    dg.set_kernel_family(family)
    try:
        _masked_check(dg, orc, case, what=f"masked G=1024 family {family}")
    finally:
        dg.set_kernel_family(0)


def test_masked_m_max_not_multiple_of_128(dg, orc):
    case = workloads.masked(G=3, M_max=200, N=96, K=384, seed=23, masked_m=[200, 77, 129])
    _masked_check(dg, orc, case)


def test_masked_config_full_size_sampled(dg, orc):
    case = workloads.masked_case()
    rng = np.random.default_rng(4)
    flat = [g * case.M_max + r for g in range(case.G) for r in
            set([0, int(case.masked_m[g]) - 1]) | set(rng.integers(0, max(1, case.masked_m[g]), 2).tolist())
            if 0 <= r < case.masked_m[g]]
    _masked_check(dg, orc, case, rows=np.array(sorted(set(flat)), np.int64), what="masked config")


def test_masked_nan_beyond_count_isolated(dg, orc):
    case = workloads.masked(G=4, M_max=256, N=128, K=256, seed=24, masked_m=[3, 200, 0, 256])
    clean = P.out_bits(P.run_masked(dg, case))
    a = case.a.copy()
    sa = case.sa.copy()
    inv = np.arange(case.M_max)[None, :] >= case.masked_m[:, None]
    a[inv] = 0x7F
    sa[inv] = np.nan
    dirty = P.out_bits(P.run_masked(dg, case, a=a, sa=sa))
    assert np.array_equal(clean[~inv], dirty[~inv])
    assert np.all(dirty[inv] == P.SENTINEL)


def test_masked_out_of_range_count_reports_layout_error(dg):
    case = workloads.masked(G=2, M_max=128, N=64, K=128, seed=25, masked_m=[10, 20])
    case.masked_m = np.array([10, 500], np.int32)
    P.run_masked(dg, case)
    assert dg.poll_device_error() == dg.DG_ERR_LAYOUT


def test_no_device_error_left(dg):
    assert dg.poll_device_error() == 0


def test_tensor_map_cache_hits_and_matches_uncached(dg, orc):
    """Repeated calls on the same buffers reuse their encoded tensor maps, and the results are
    bit-identical with the cache on and off (and match the oracle)."""
    case = workloads.dense(200, 1000, 640, seed=801)
    a, b = P.to_dev_u8(case.a), P.to_dev_u8(case.b)
    sfa, sfb = dg.sfa_mn_major(P.to_dev_f32(case.sa)), P.to_dev_f32(case.sb)
    d = P.sentinel_out((case.M, case.N))
    dg.dg_gemm_fp8_fp8_bf16_nt(a, sfa, b, sfb, d)
    torch.cuda.synchronize()
    first = P.out_bits(d)
    h0, m0 = dg.tensor_map_cache_stats()
    for _ in range(3):
        dg.dg_gemm_fp8_fp8_bf16_nt(a, sfa, b, sfb, d)
    torch.cuda.synchronize()
    h1, m1 = dg.tensor_map_cache_stats()
    assert h1 - h0 >= 6 and m1 == m0, (h0, m0, h1, m1)
    assert np.array_equal(P.out_bits(d), first)
    prev = dg.set_tensor_map_cache(False)
    try:
        d.view(torch.int16).fill_(-1)
        dg.dg_gemm_fp8_fp8_bf16_nt(a, sfa, b, sfb, d)
        torch.cuda.synchronize()
        uncached = P.out_bits(d)
    finally:
        dg.set_tensor_map_cache(prev)
    assert np.array_equal(uncached, first)
    ref = orc.gemm_dense(case.a, case.sa, case.b, case.sb)
    P.check(first, ref, "cached maps")
    assert dg.poll_device_error() == 0
