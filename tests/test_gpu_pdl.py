"""Programmatic dependent launch: with it on, back-to-back GEMMs may be scheduled while the
previous one finishes, and every kernel waits (griddepcontrol.wait) before touching global
memory.  These tests launch dependent sequences with no synchronisation in between and check
that the results are bit-identical to the same launches made one at a time: a later GEMM
overwriting the earlier one's output (write after write), a GEMM whose A operand is the earlier
GEMM's output reinterpreted as e4m3 bytes (read after write), and a long mixed sequence of the
three kernel families."""
from __future__ import annotations

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fp8_block_scaled_tma_b200 as mod
    mod.set_kernel_family(0)
    mod.set_config_override(0, 0, 0)
    prev = mod.set_pdl(True)
    yield mod
    mod.set_pdl(prev)
    mod.set_kernel_family(0)


def _dev(case):
    import fp8_block_scaled_tma_b200 as mod
    a = torch.from_numpy(case.a).cuda()
    b = torch.from_numpy(case.b).cuda()
    sfa = mod.sfa_mn_major(torch.from_numpy(case.sa).cuda())
    sfb = torch.from_numpy(case.sb).cuda()
    return a, sfa, b, sfb


def _bits(t):
    return t.view(torch.int16).cpu()


def test_write_after_write(dg):
    """A long GEMM then a short one into the same output: the short one's result must win."""
    big = _dev(workloads.dense(4096, 2112, 7168, seed=301))
    small = _dev(workloads.dense(4096, 2112, 256, seed=302))
    ref = torch.empty(4096, 2112, dtype=torch.bfloat16, device="cuda")
    dg.dg_gemm_fp8_fp8_bf16_nt(*small, ref)
    torch.cuda.synchronize()
    d = torch.zeros(4096, 2112, dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        dg.dg_gemm_fp8_fp8_bf16_nt(*big, d)
        dg.dg_gemm_fp8_fp8_bf16_nt(*small, d)
    torch.cuda.synchronize()
    assert dg.poll_device_error() == 0
    assert torch.equal(_bits(d), _bits(ref))


def _pm_one_codes(rows, k, gen):
    """e4m3 codes of +1 (0x38) and -1 (0xB8)."""
    bits = torch.randint(0, 2, (rows, k), generator=gen, dtype=torch.uint8)
    return (0x38 + 0x80 * bits).to(torch.uint8).cuda()


@pytest.mark.parametrize("M1,family2", [(4096, 0), (4096, 3), (512, 1)])
def test_read_after_write(dg, M1, family2):
    """GEMM 2 reads GEMM 1's bf16 output, reinterpreted as e4m3 bytes, as its A operand.
    GEMM 1 sums 128 products of +-1 with unit scales, so D1 holds even integers of magnitude
    below 128; their bf16 bytes have a zero last mantissa bit and a small exponent, so no byte
    is an e4m3 NaN code and every byte is a finite operand for GEMM 2."""
    N1 = 1024  # D1 row = 2048 bytes = one e4m3 row of K2 = 2048
    gen = torch.Generator().manual_seed(303)
    a1 = _pm_one_codes(M1, 128, gen)
    b1 = _pm_one_codes(N1, 128, gen)
    sfa1 = dg.sfa_mn_major(torch.ones(M1, 1, device="cuda"))
    sfb1 = torch.ones(N1 // 128, 1, device="cuda")
    g1 = (a1, sfa1, b1, sfb1)
    case2 = workloads.dense(64, 768, 2 * N1, seed=304)
    _, _, b2, sfb2 = _dev(case2)
    sfa2 = dg.sfa_mn_major(torch.ones(M1, 2 * N1 // 128, device="cuda") * 1e-3)
    d1 = torch.zeros(M1, N1, dtype=torch.bfloat16, device="cuda")
    d2 = torch.zeros(M1, 768, dtype=torch.bfloat16, device="cuda")
    a2 = d1.view(torch.uint8).view(M1, 2 * N1)  # aliases d1
    dg.set_kernel_family(family2)
    try:
        for _ in range(3):
            d1.zero_()
            torch.cuda.synchronize()
            dg.dg_gemm_fp8_fp8_bf16_nt(*g1, d1)
            dg.dg_gemm_fp8_fp8_bf16_nt(a2, sfa2, b2, sfb2, d2)  # no sync in between
        torch.cuda.synchronize()
        assert dg.poll_device_error() == 0
        # the same second GEMM on a settled copy of D1
        a2_copy = a2.clone()
        ref = torch.zeros_like(d2)
        dg.dg_gemm_fp8_fp8_bf16_nt(a2_copy, sfa2, b2, sfb2, ref)
        torch.cuda.synchronize()
    finally:
        dg.set_kernel_family(0)
    assert torch.count_nonzero(a2_copy) > 0
    assert not bool(((a2_copy & 0x7F) == 0x7F).any())  # no e4m3 NaN code
    assert torch.equal(_bits(d2), _bits(ref))


def test_long_mixed_sequence_matches_one_at_a_time(dg):
    shapes = [(64, 2112, 7168), (4096, 448, 1024), (128, 7168, 2048), (300, 1000, 640),
              (4096, 2112, 1536), (1, 256, 1280)]
    cases = [_dev(workloads.dense(M, N, K, seed=310 + i)) for i, (M, N, K) in enumerate(shapes)]
    outs = [torch.zeros(M, N, dtype=torch.bfloat16, device="cuda") for (M, N, K) in shapes]
    refs = [torch.zeros_like(o) for o in outs]
    for c, r in zip(cases, refs):
        dg.dg_gemm_fp8_fp8_bf16_nt(*c, r)
        torch.cuda.synchronize()
    for rnd in range(4):
        for c, o in zip(cases, outs):
            dg.dg_gemm_fp8_fp8_bf16_nt(*c, o)
    torch.cuda.synchronize()
    assert dg.poll_device_error() == 0
    for o, r in zip(outs, refs):
        assert torch.equal(_bits(o), _bits(r))


def test_switch_off_gives_same_results(dg):
    case = _dev(workloads.dense(128, 4096, 7168, seed=320))
    on = torch.zeros(128, 4096, dtype=torch.bfloat16, device="cuda")
    off = torch.zeros_like(on)
    dg.dg_gemm_fp8_fp8_bf16_nt(*case, on)
    prev = dg.set_pdl(False)
    try:
        dg.dg_gemm_fp8_fp8_bf16_nt(*case, off)
    finally:
        dg.set_pdl(prev)
    torch.cuda.synchronize()
    assert torch.equal(_bits(on), _bits(off))
