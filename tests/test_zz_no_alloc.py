"""The allocation-free dense entry point, dg_gemm_fp8_fp8_bf16_nt_noalloc.

Some callers cannot allocate device memory while they work -- a serving loop whose memory is
planned up front, an operator inside another runtime that only receives its inputs and outputs,
a latency-critical thread on which cudaMalloc could synchronise the device -- so they cannot
hand the stream-K kernel the workspace it needs.  This entry point runs that kernel with its
scratch in an array built into the library.  The test calls it through the C ABI twice in a
row and checks both results against the ordinary entry point's, within the parity tolerance the
other tests use (per element 2 bf16 ulp + 1e-3 sum |sa a| |sb b|, per matrix 1e-5); the two
calls must also agree bit for bit, since the second starts from what the first left in the
shared array.  It lives in a file of its own, collected last, and passes alone in a fresh
process as well as after the other tests.
"""
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
    return mod


def _noalloc(dg, a, sfa, b, sfb, d, M, N, K):
    """One call through the C ABI (no binding-side checks in between)."""
    return dg.lib.dg_gemm_fp8_fp8_bf16_nt_noalloc(a.data_ptr(), sfa.data_ptr(), b.data_ptr(),
                                                  sfb.data_ptr(), d.data_ptr(), M, N, K,
                                                  torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_the_allocating_entry_point_twice(dg):
    import oracle
    oracle.build()
    M, N, K = 64, 7168, 4096
    case = workloads.dense(M, N, K, seed=4242, a_std=1.0, b_std=0.02)
    a, b = P.to_dev_u8(case.a), P.to_dev_u8(case.b)
    sfa, sfb = dg.sfa_mn_major(P.to_dev_f32(case.sa)), P.to_dev_f32(case.sb)
    # the existing entry point (automatic kernel choice, no workspace)
    d_ref = P.sentinel_out((M, N))
    dg.dg_gemm_fp8_fp8_bf16_nt(a, sfa, b, sfb, d_ref)
    torch.cuda.synchronize()
    ref_bits = P.out_bits(d_ref)
    mag = oracle.gemm_dense(case.a, case.sa, case.b, case.sb).mag  # the tolerance's magnitude term
    results = []
    for call in range(2):
        d = P.sentinel_out((M, N))
        assert _noalloc(dg, a, sfa, b, sfb, d, M, N, K) == dg.DG_OK
        torch.cuda.synchronize()
        got = P.out_bits(d)
        assert not np.any(got == P.SENTINEL), f"call {call}: an output was not written"
        r = P.compare(got, ref_bits, mag)
        assert r["n_bad"] == 0, f"call {call}: {r}"
        assert r["diff"] <= P.DIFF_MAX, f"call {call}: {r}"
        results.append(got)
    assert np.array_equal(results[0], results[1])
    assert dg.get_last_launch()["family"] == 5
    assert dg.poll_device_error() == 0


def test_noalloc_rejects_what_it_cannot_take(dg):
    """Beyond 64 tokens, or for shapes the kernel does not take, DG_ERR_UNSUPPORTED with
    nothing written; M == 0 is a no-op."""
    for (M, N, K) in [(65, 2112, 4096), (64, 1024, 1024)]:
        case = workloads.dense(M, N, K, seed=M + N)
        a, b = P.to_dev_u8(case.a), P.to_dev_u8(case.b)
        sfa, sfb = dg.sfa_mn_major(P.to_dev_f32(case.sa)), P.to_dev_f32(case.sb)
        d = P.sentinel_out((M, N))
        assert _noalloc(dg, a, sfa, b, sfb, d, M, N, K) == dg.DG_ERR_UNSUPPORTED
        torch.cuda.synchronize()
        assert np.all(P.out_bits(d) == P.SENTINEL)
    z = torch.zeros(16, dtype=torch.uint8, device="cuda")
    assert dg.lib.dg_gemm_fp8_fp8_bf16_nt_noalloc(z.data_ptr(), z.data_ptr(), z.data_ptr(), z.data_ptr(),
                                                  z.data_ptr(), 0, 256, 128, None) == dg.DG_OK
