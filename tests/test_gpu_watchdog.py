"""The pipeline watchdog: with the fault-injection hook on, the MMA issuer waits on a barrier
that nothing signals; after a short wait limit the kernels give up, report DG_ERR_TIMEOUT
through the device error word, drain their in-flight copies and MMAs, free tensor memory and
return -- and the CUDA context stays usable (the next normal call is correct).  Nothing here
faults, traps or hangs the GPU: every wait in the kernels is bounded."""
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
    mod.set_kernel_family(0)
    mod.set_config_override(0, 0, 0)
    assert mod.poll_device_error() == 0
    yield mod
    mod.set_fault_injection(0)
    mod.set_wait_timeout_ns(0)
    mod.set_kernel_family(0)


@pytest.fixture(scope="module")
def orc():
    import oracle
    oracle.build()
    return oracle


@pytest.mark.parametrize("family,M,N,K", [
    (1, 1024, 2048, 4096),   # one-CTA persistent kernel
    (2, 1024, 2048, 4096),   # CTA-pair kernel
    (3, 128, 2048, 8192),    # split-K cluster kernel
    (4, 64, 2048, 8192),     # swapped-operand kernel
])
def test_wait_limit_reports_timeout_and_context_survives(dg, orc, family, M, N, K):
    case = workloads.dense(M, N, K, seed=family)
    prev = dg.set_wait_timeout_ns(1_000_000)  # 1 ms
    dg.set_kernel_family(family)
    dg.set_fault_injection(1)
    try:
        P.run_dense(dg, case)
        status = dg.poll_device_error()
        assert dg.get_last_launch()["family"] == family
    finally:
        dg.set_fault_injection(0)
        dg.set_wait_timeout_ns(prev)
        dg.set_kernel_family(0)
    assert status == dg.DG_ERR_TIMEOUT
    # the error word was cleared by the poll, and the next call is correct
    small = workloads.small_dense()
    got = P.out_bits(P.run_dense(dg, small))
    ref = orc.gemm_dense(small.a, small.sa, small.b, small.sb)
    P.check(got, ref, "after timeout")
    assert dg.poll_device_error() == 0


def test_masked_pair_timeout(dg, orc):
    case = workloads.masked(G=4, M_max=256, N=512, K=2048, seed=5, masked_m=[256, 100, 0, 200])
    prev = dg.set_wait_timeout_ns(1_000_000)
    dg.set_fault_injection(1)
    try:
        got = P.out_bits(P.run_masked(dg, case))
        status = dg.poll_device_error()
    finally:
        dg.set_fault_injection(0)
        dg.set_wait_timeout_ns(prev)
    assert status == dg.DG_ERR_TIMEOUT
    # rows the call must never write stay untouched even when the pipeline gave up
    inv = np.arange(case.M_max)[None, :] >= case.masked_m[:, None]
    assert np.all(got[inv] == P.SENTINEL)
    got = P.out_bits(P.run_masked(dg, case))
    assert dg.poll_device_error() == 0
    ref = orc.gemm_masked(case.a, case.sa, case.b, case.sb, case.masked_m)
    P.check(got, ref, "masked after timeout", sel=~inv)
