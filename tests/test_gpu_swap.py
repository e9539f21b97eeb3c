"""GPU parity of the swapped-operand kernel (dense, M <= 128: B rows on the MMA's 128-lane side,
the tokens on its N side, K split over a cluster) against the oracle: token tiles of 32, 64 and
128, one or two 128-row blocks of B per tile, every split count, FP4 B, ragged shapes, the
full-size decode shapes on sampled rows, and bit-identical repeats."""
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
    mod.set_kernel_family(0)
    yield mod
    mod.set_config_override(0, 0)
    mod.set_num_sms(0)
    mod.set_kernel_family(0)


@pytest.fixture(scope="module")
def orc():
    import oracle
    oracle.build()
    return oracle


def _check(dg, orc, case, what, fp4=False, rows=None):
    got = P.out_bits(P.run_dense_fp4(dg, case) if fp4 else P.run_dense(dg, case))
    b = orc.e2m1_to_e4m3(case.b) if fp4 else case.b
    if rows is None:
        assert not np.any(got == P.SENTINEL)
        ref = orc.gemm_dense(case.a, case.sa, b, case.sb)
        r = P.assert_close(got, ref.bits, ref.mag, what, acc=ref.acc)
    else:
        ref = orc.gemm_dense(case.a, case.sa, b, case.sb, rows=rows)
        r = P.assert_close(got[rows], ref.bits, ref.mag, what, acc=ref.acc)
    assert dg.poll_device_error() == 0
    return r


def _forced(dg, fn, block_n=0, splits=0):
    dg.set_kernel_family(4)
    dg.set_config_override(block_n, 0, splits)
    try:
        out = fn()
        ll = dg.get_last_launch()
    finally:
        dg.set_config_override(0, 0)
        dg.set_kernel_family(0)
    assert ll["family"] == 4
    return out, ll


@pytest.mark.parametrize("M,N,K", [
    (1, 8, 128),          # one token, one 8-column output block, one K block
    (7, 136, 384),        # token tile 32, N tail of 8, 3 K blocks
    (32, 256, 256),
    (33, 1000, 640),      # token tile 64, ragged N
    (64, 2112, 7168),     # N tail block of 64 rows, many splits
    (65, 520, 1664),      # token tile 128, 13 K blocks
    (100, 4096, 512),
    (128, 7168, 2048),
])
def test_swap_forced(dg, orc, M, N, K):
    case = workloads.dense(M, N, K, seed=M + 5 * N + K, a_std=1.0, b_std=0.02)
    r, _ = _forced(dg, lambda: _check(dg, orc, case, f"swap {M}x{N}x{K}"))
    assert r["excess"] < 2e-5, r


@pytest.mark.parametrize("M", [20, 64, 128])
@pytest.mark.parametrize("N", [384, 2112])
def test_swap_two_row_blocks(dg, orc, M, N):
    """R = 2 (256 B rows per tile, two MMAs per K step); N = 384 and 2112 leave the last tile
    with one real 128-row block."""
    case = workloads.dense(M, N, 1024, seed=M + N)
    _, ll = _forced(dg, lambda: _check(dg, orc, case, f"swap R=2 {M}x{N}"), block_n=256)
    assert ll["block_n"] == 256


@pytest.mark.parametrize("splits", [1, 2, 3, 5, 8])
def test_swap_every_split_count(dg, orc, splits):
    case = workloads.dense(48, 1024, 2304, seed=splits + 40)
    _, ll = _forced(dg, lambda: _check(dg, orc, case, f"swap S={splits}"), splits=splits)
    assert ll["splits"] == splits


@pytest.mark.parametrize("M,N,K,block_n", [
    (1, 256, 256, 0), (40, 1000, 1280, 0), (128, 2112, 2048, 0), (64, 768, 1024, 256),
])
def test_swap_fp4(dg, orc, M, N, K, block_n):
    case = workloads.with_fp4_b(workloads.dense(M, N, K, seed=M + N), seed=K)
    _forced(dg, lambda: _check(dg, orc, case, f"swap fp4 {M}x{N}x{K}", fp4=True), block_n=block_n)


@pytest.mark.parametrize("M", [64, 128])
@pytest.mark.parametrize("N,K", [(2112, 7168), (24576, 1536), (7168, 16384), (4096, 7168), (7168, 2048)])
def test_swap_decode_shapes_sampled(dg, orc, M, N, K):
    """The full-size decode shapes of the DeepSeek-V3 projections, forced onto this kernel, and
    in auto mode (which takes it for M <= 64 when one 128-row block of B per tile fits in one
    wave)."""
    case = workloads.dense(M, N, K, seed=M * 3 + N + K, a_std=1.0, b_std=0.02)
    rows = P.sample_rows(M, 16, seed=M + N)
    _forced(dg, lambda: _check(dg, orc, case, f"swap {M}x{N}x{K}", rows=rows))
    _check(dg, orc, case, f"auto {M}x{N}x{K}", rows=rows)
    ll = dg.get_last_launch()
    assert (ll["family"] == 4) == (M <= 64 and N <= 148 * 128), ll
    if ll["family"] == 4:
        assert ll["block_n"] == 128


def test_swap_sm_cap(dg, orc):
    case = workloads.dense(64, 2048, 4096, seed=91)
    prev = dg.set_num_sms(24)
    try:
        _, ll = _forced(dg, lambda: _check(dg, orc, case, "swap cap 24"))
    finally:
        dg.set_num_sms(prev)
    assert ll["grid"] <= 24


def test_swap_deterministic(dg):
    case = workloads.dense(96, 2112, 7168, seed=92)
    (a, b), ll = _forced(dg, lambda: (P.out_bits(P.run_dense(dg, case)),
                                      P.out_bits(P.run_dense(dg, case))))
    assert ll["splits"] > 1
    assert np.array_equal(a, b)


def test_swap_family_leaves_larger_m_to_the_others(dg, orc):
    """Family 4 applies to dense M <= 128; a larger M runs as in auto mode."""
    case = workloads.dense(129, 256, 256, seed=93)
    dg.set_kernel_family(4)
    try:
        _check(dg, orc, case, "M=129 under family 4")
        assert dg.get_last_launch()["family"] != 4
    finally:
        dg.set_kernel_family(0)
