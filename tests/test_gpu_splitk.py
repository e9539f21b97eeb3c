"""GPU parity of the split-K cluster kernel (dense; the K blocks of a tile split over up to 8
CTAs that reduce their fp32 partials through distributed shared memory) against the oracle."""
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


def _check(dg, orc, case, what):
    got = P.out_bits(P.run_dense(dg, case))
    assert not np.any(got == P.SENTINEL)
    ref = orc.gemm_dense(case.a, case.sa, case.b, case.sb)
    r = P.assert_close(got, ref.bits, ref.mag, what, acc=ref.acc)
    assert dg.poll_device_error() == 0
    return r


@pytest.mark.parametrize("M,N,K", [
    (64, 2112, 7168),    # many splits per tile, N tail block of 64 rows
    (128, 7168, 2048),
    (1, 256, 1280),      # one valid row
    (100, 1000, 1664),   # ragged M and N, 13 K blocks (odd per-split counts)
    (256, 512, 384),     # 3 K blocks, two 128-row tiles
    (200, 4096, 512),
])
def test_splitk_forced(dg, orc, M, N, K):
    case = workloads.dense(M, N, K, seed=M + 3 * N + K, a_std=1.0, b_std=0.02)
    dg.set_kernel_family(3)
    try:
        r = _check(dg, orc, case, f"split-K {M}x{N}x{K}")
        assert dg.get_last_launch()["family"] == 3
    finally:
        dg.set_kernel_family(0)
    assert r["excess"] < 2e-5


@pytest.mark.parametrize("bn", [64, 96, 128, 160, 192, 224, 256])
def test_splitk_every_block_n(dg, orc, bn):
    case = workloads.dense(96, 1040, 2048, seed=bn + 7)
    dg.set_kernel_family(3)
    dg.set_config_override(bn, 0)
    try:
        _check(dg, orc, case, f"split-K BN={bn}")
        ll = dg.get_last_launch()
        assert ll["block_n"] == bn and ll["family"] == 3
    finally:
        dg.set_config_override(0, 0)
        dg.set_kernel_family(0)


def test_splitk_auto_selected_for_small_m(dg, orc):
    """Auto mode: 128 < M <= 256 runs split-K (M <= 128 takes the swapped-operand kernel)."""
    case = workloads.dense(200, 4096, 7168, seed=71, a_std=1.0, b_std=0.02)
    _check(dg, orc, case, "auto small M")
    ll = dg.get_last_launch()
    assert ll["family"] == 3 and ll["splits"] > 1


def test_splitk_sm_cap(dg, orc):
    """With 20 SMs the chooser must fit tiles x splits into 20 CTAs."""
    case = workloads.dense(128, 1024, 4096, seed=72)
    prev = dg.set_num_sms(20)
    dg.set_kernel_family(3)
    try:
        _check(dg, orc, case, "split-K cap 20")
        assert dg.get_last_launch()["grid"] <= 20
    finally:
        dg.set_kernel_family(0)
        dg.set_num_sms(prev)


def test_splitk_deterministic(dg):
    """The reduction sums the partials in a fixed order: repeated calls are bit-identical."""
    case = workloads.dense(128, 2112, 7168, seed=73)
    dg.set_kernel_family(3)
    try:
        a = P.out_bits(P.run_dense(dg, case))
        b = P.out_bits(P.run_dense(dg, case))
        assert dg.get_last_launch()["splits"] > 1
    finally:
        dg.set_kernel_family(0)
    assert np.array_equal(a, b)
