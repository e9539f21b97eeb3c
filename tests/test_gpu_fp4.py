"""GPU parity of the FP8 x FP4 GEMMs (e4m3 A, packed E2M1 B) against the oracle: the oracle
expands B's E2M1 values into e4m3 codes of the same values (exact: every E2M1 value is an e4m3
value) and runs its FP8 GEMM, so the expected result is the block-scaled formula with B's FP4
values.  Every kernel family and layout is covered: the one-CTA, CTA-pair and split-K kernels
(dense), contiguous and masked grouped layouts, every BN, ragged shapes, and full-size
decode and prefill shapes on sampled rows."""
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
    assert mod.poll_device_error() == 0
    yield mod
    mod.set_config_override(0, 0)
    mod.set_num_sms(0)
    mod.set_kernel_family(0)


@pytest.fixture(scope="module")
def orc():
    import oracle
    oracle.build()
    return oracle


def _dense(dg, orc, case, what, rows=None):
    got = P.out_bits(P.run_dense_fp4(dg, case))
    b = orc.e2m1_to_e4m3(case.b)
    if rows is None:
        ref = orc.gemm_dense(case.a, case.sa, b, case.sb)
        r = P.assert_close(got, ref.bits, ref.mag, what, acc=ref.acc)
    else:
        ref = orc.gemm_dense(case.a, case.sa, b, case.sb, rows=rows)
        r = P.assert_close(got[rows], ref.bits, ref.mag, what, acc=ref.acc)
    assert dg.poll_device_error() == 0
    return r


@pytest.mark.parametrize("family", [0, 1, 2, 3])
@pytest.mark.parametrize("M,N,K", [
    (1, 8, 128),          # one row, one 8-column output block, one K block
    (7, 136, 384),        # ragged M and N, 3 K blocks
    (130, 264, 256),      # two M tiles, N tail of 8
    (300, 1000, 640),     # ragged everywhere
    (256, 2112, 1024),    # N tail block of 64 rows
])
def test_fp4_dense_families(dg, orc, family, M, N, K):
    case = workloads.with_fp4_b(workloads.dense(M, N, K, seed=M + 3 * N + K), seed=M + N)
    dg.set_kernel_family(family)
    try:
        r = _dense(dg, orc, case, f"fp4 family {family} {M}x{N}x{K}")
    finally:
        dg.set_kernel_family(0)
    assert r["excess"] < 2e-5, r


@pytest.mark.parametrize("bn", [32, 64, 96, 128, 160, 192, 224, 256])
def test_fp4_every_block_n(dg, orc, bn):
    case = workloads.with_fp4_b(workloads.dense(300, 1000, 640, seed=bn), seed=bn + 1)
    dg.set_kernel_family(1)
    dg.set_config_override(bn, 0)
    try:
        _dense(dg, orc, case, f"fp4 BN={bn}")
        assert dg.get_last_launch()["block_n"] == bn
    finally:
        dg.set_config_override(0, 0)
        dg.set_kernel_family(0)


@pytest.mark.parametrize("splits", [2, 5, 8])
def test_fp4_splitk_forced(dg, orc, splits):
    case = workloads.with_fp4_b(workloads.dense(64, 512, 2048, seed=splits), seed=splits + 9)
    dg.set_kernel_family(3)
    dg.set_config_override(0, 0, splits)
    try:
        _dense(dg, orc, case, f"fp4 split-K {splits}")
        assert dg.get_last_launch()["splits"] == splits
    finally:
        dg.set_config_override(0, 0)
        dg.set_kernel_family(0)


def test_fp4_equals_fp8_of_same_values(dg, orc):
    """The FP4 call and the FP8 call on B's values expanded to e4m3 codes agree within the
    parity tolerance (the products are exact either way)."""
    case = workloads.with_fp4_b(workloads.dense(256, 768, 1024, seed=5), seed=6)
    got4 = P.out_bits(P.run_dense_fp4(dg, case))
    import dataclasses
    case8 = dataclasses.replace(case, b=orc.e2m1_to_e4m3(case.b))
    got8 = P.out_bits(P.run_dense(dg, case8))
    ref = orc.gemm_dense(case8.a, case8.sa, case8.b, case8.sb)
    P.check(got4, ref, "fp4")
    P.check(got8, ref, "fp8 of the same values")
    assert np.mean(got4 == got8) > 0.99


@pytest.mark.parametrize("M", [64, 128, 4096])
def test_fp4_decode_and_prefill_shapes_sampled(dg, orc, M):
    """Full-size shapes of the DeepSeek-V3 projections (N x K = 7168 x 2048 and 2112 x 7168)
    on sampled rows."""
    for N, K in [(7168, 2048), (2112, 7168)]:
        case = workloads.with_fp4_b(workloads.dense(M, N, K, seed=M + N), seed=K)
        rows = P.sample_rows(M, 8, seed=M)
        _dense(dg, orc, case, f"fp4 {M}x{N}x{K}", rows=rows)


def test_fp4_contiguous(dg, orc):
    case = workloads.with_fp4_b(
        workloads.contiguous(G=4, N=384, K=512, seed=21, counts=[1, 130, 0, 300]), seed=22)
    got = P.out_bits(P.run_contiguous_fp4(dg, case))
    ref = orc.gemm_contiguous(case.a, case.sa, orc.e2m1_to_e4m3(case.b), case.sb, case.m_indices)
    pad = case.m_indices < 0
    assert np.all(got[pad] == P.SENTINEL), "a padding row was written"
    P.check(got, ref, "fp4 contiguous", sel=~pad)
    assert dg.poll_device_error() == 0


@pytest.mark.parametrize("family", [1, 2])
def test_fp4_masked(dg, orc, family):
    case = workloads.with_fp4_b(
        workloads.masked(G=4, M_max=256, N=512, K=768, seed=31, masked_m=[256, 0, 1, 200]),
        seed=32)
    dg.set_kernel_family(family)
    try:
        got = P.out_bits(P.run_masked_fp4(dg, case))
    finally:
        dg.set_kernel_family(0)
    ref = orc.gemm_masked(case.a, case.sa, orc.e2m1_to_e4m3(case.b), case.sb, case.masked_m)
    inv = np.arange(case.M_max)[None, :] >= case.masked_m[:, None]
    assert np.all(got[inv] == P.SENTINEL), "a row beyond masked_m was written"
    P.check(got, ref, f"fp4 masked family {family}", sel=~inv)
    assert dg.poll_device_error() == 0


def test_fp4_b_alignment_enforced(dg):
    case = workloads.with_fp4_b(workloads.dense(128, 256, 256, seed=1), seed=2)
    a = P.to_dev_u8(case.a)
    buf = torch.zeros(case.b.size + 32, dtype=torch.uint8, device="cuda")
    b16 = buf[16:16 + case.b.size]               # 16- but not 32-byte aligned
    sfa = dg.sfa_mn_major(P.to_dev_f32(case.sa))
    sfb = P.to_dev_f32(case.sb)
    d = P.sentinel_out((128, 256))
    r = dg.lib.dg_gemm_fp8_fp4_bf16_nt(a.data_ptr(), sfa.data_ptr(), b16.data_ptr(),
                                       sfb.data_ptr(), d.data_ptr(), 128, 256, 256, None)
    assert r == dg.DG_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert np.all(P.out_bits(d) == P.SENTINEL)
