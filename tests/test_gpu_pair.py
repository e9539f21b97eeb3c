"""GPU parity of the CTA-pair kernels (tcgen05 cta_group::2, 256-row tiles, K-block-pair TMA
boxes) and of the one-CTA kernels forced on the same cases, against the CPU oracle."""
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


def _dense(dg, orc, case, what):
    got = P.out_bits(P.run_dense(dg, case))
    ref = orc.gemm_dense(case.a, case.sa, case.b, case.sb)
    r = P.assert_close(got, ref.bits, ref.mag, what, acc=ref.acc)
    assert dg.poll_device_error() == 0
    return r


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("M,N,K", [
    (256, 512, 384),     # 3 K blocks: the last TMA box holds one real K block
    (300, 1000, 640),    # ragged M and N
    (1, 256, 256),       # the odd CTA of the pair has no valid row
    (520, 2112, 1024),   # N tail block of 64 rows
    (4096, 448, 256),
])
def test_dense_pair_modes(dg, orc, mode, M, N, K):
    case = workloads.dense(M, N, K, seed=M + N + K + mode, a_std=1.0, b_std=0.02)
    dg.set_kernel_family(mode)
    try:
        r = _dense(dg, orc, case, f"mode {mode} {M}x{N}x{K}")
    finally:
        dg.set_kernel_family(0)
    assert r["excess"] < 2e-5


@pytest.mark.parametrize("bn", [128, 160, 192, 224, 256])
def test_dense_pair_every_block_n(dg, orc, bn):
    case = workloads.dense(600, 1040, 1280, seed=bn + 1)
    dg.set_kernel_family(2)
    dg.set_config_override(bn, 0)
    try:
        _dense(dg, orc, case, f"pair BN={bn}")
        ll = dg.get_last_launch()
        assert ll["block_n"] == bn and ll["grid"] % 2 == 0
    finally:
        dg.set_config_override(0, 0)
        dg.set_kernel_family(0)


def test_dense_pair_two_stages_and_sm_cap(dg, orc):
    """3 CTA pairs (7 SMs allowed) walk many tiles with only 2 pipeline stages."""
    case = workloads.dense(1024, 2048, 1536, seed=3)
    prev = dg.set_num_sms(7)
    dg.set_kernel_family(2)
    dg.set_config_override(128, 2)
    try:
        _dense(dg, orc, case, "pair cap 7, 2 stages")
        ll = dg.get_last_launch()
        assert ll["grid"] == 6 and ll["stages"] == 2
    finally:
        dg.set_config_override(0, 0)
        dg.set_kernel_family(0)
        dg.set_num_sms(prev)


def _masked(dg, orc, case, what):
    got = P.out_bits(P.run_masked(dg, case))
    inv = np.arange(case.M_max)[None, :] >= case.masked_m[:, None]
    assert np.all(got[inv] == P.SENTINEL), "a row beyond masked_m was written"
    ref = orc.gemm_masked(case.a, case.sa, case.b, case.sb, case.masked_m)
    P.check(got, ref, what, sel=~inv)
    assert dg.poll_device_error() == 0


@pytest.mark.parametrize("mode", [1, 2])
def test_masked_pair_edge_counts(dg, orc, mode):
    case = workloads.masked(G=6, M_max=256, N=136, K=256, seed=31,
                            masked_m=[0, 1, 127, 128, 129, 256])
    dg.set_kernel_family(mode)
    try:
        _masked(dg, orc, case, f"masked mode {mode}")
    finally:
        dg.set_kernel_family(0)


@pytest.mark.parametrize("mode", [1, 2])
def test_masked_pair_two_tiles_per_group(dg, orc, mode):
    """M_max = 512: groups with more than one 256-row pair tile, plus an odd K-block count."""
    case = workloads.masked(G=3, M_max=512, N=192, K=384, seed=32, masked_m=[512, 257, 300])
    dg.set_kernel_family(mode)
    try:
        _masked(dg, orc, case, f"masked 512 mode {mode}")
    finally:
        dg.set_kernel_family(0)


def test_masked_pair_m_max_200(dg, orc):
    case = workloads.masked(G=4, M_max=200, N=256, K=512, seed=33, masked_m=[200, 0, 64, 199])
    dg.set_kernel_family(2)
    try:
        _masked(dg, orc, case, "masked 200 pair")
    finally:
        dg.set_kernel_family(0)


def test_pair_and_single_agree_closely(dg):
    """Both kernel families on the same inputs: identical up to fp32 accumulation order."""
    case = workloads.dense(512, 1024, 2048, seed=9)
    dg.set_kernel_family(1)
    a = P.bits_to_f64(P.out_bits(P.run_dense(dg, case)))
    dg.set_kernel_family(2)
    b = P.bits_to_f64(P.out_bits(P.run_dense(dg, case)))
    dg.set_kernel_family(0)
    assert np.max(np.abs(a - b) / (np.abs(a) + 1e-3)) < 2 ** -7
