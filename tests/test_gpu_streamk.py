"""GPU parity of the stream-K swapped-operand kernel (dense, M <= 64: every SM takes an equal
share of the K blocks, the partials of a tile meet in the caller's workspace and the last
contributor adds them in K order; kernel family 5, opt-in) against the oracle: the decode
shapes at full size, ragged sizes, one unit per CTA (148 contributors of one tile; 148 tiles of
one contributor), edge-value inputs, bit-identical repeats, the workspace's counters back at
zero after each call, the workspace checks, and the watchdog path."""
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


def _counters(dg, ws, M, N, K):
    """The workspace's per-tile counters (they follow the partial slots)."""
    n_tiles = -(-N // 128)
    sms = dg.get_num_sms()
    tn = 32 if M <= 32 else 64
    off = sms * 2 * tn * 128 * 4
    return ws[off:off + 4 * n_tiles].view(torch.int32).cpu().numpy()


def _run(dg, orc, case, what, family=5):
    ws = dg.workspace_for(case.M, case.N, case.K)
    assert ws is not None, "the stream-K kernel does not apply to this shape"
    dg.set_kernel_family(family)
    try:
        got = P.out_bits(P.run_dense(dg, case, workspace=ws))
        ll = dg.get_last_launch()
    finally:
        dg.set_kernel_family(0)
    assert ll["family"] == 5, ll
    assert not np.any(got == P.SENTINEL)
    ref = orc.gemm_dense(case.a, case.sa, case.b, case.sb)
    r = P.check(got, ref, what)
    assert dg.poll_device_error() == 0
    assert np.all(_counters(dg, ws, case.M, case.N, case.K) == 0), "tile counters not back at zero"
    return got, ws, r


@pytest.mark.parametrize("M,N,K", [
    (64, 2112, 7168), (64, 7168, 16384), (64, 4096, 7168), (64, 7168, 2048),   # decode shapes
    (1, 2112, 7168), (7, 136, 18432), (33, 2112, 2048), (64, 1000, 4096), (48, 7168, 1024),
])
def test_streamk_parity(dg, orc, M, N, K):
    case = workloads.dense(M, N, K, seed=M + N + K, a_std=1.0, b_std=0.02)
    _run(dg, orc, case, f"stream-K {M}x{N}x{K}")


def test_streamk_one_unit_per_cta(dg, orc):
    """148 K blocks of one tile: every CTA takes one unit, the tile has 148 contributors; and
    148 tiles of one K block: every tile has one contributor."""
    sms = dg.get_num_sms()
    _run(dg, orc, workloads.dense(3, 128, 128 * sms, seed=1), "one tile, every CTA")
    _run(dg, orc, workloads.dense(5, 128 * sms, 128, seed=2), "every CTA its own tile")


@pytest.mark.parametrize("pattern", workloads.EDGE_PATTERNS)
def test_streamk_edge_values(dg, orc, pattern):
    case = workloads.edge_dense(pattern, 40, 2112, 4096, seed=301 + workloads.EDGE_PATTERNS.index(pattern))
    ws = dg.workspace_for(case.M, case.N, case.K)
    dg.set_kernel_family(5)
    try:
        got = P.out_bits(P.run_dense(dg, case, workspace=ws))
    finally:
        dg.set_kernel_family(0)
    ref = orc.gemm_dense(case.a, case.sa, case.b, case.sb)
    P.check(got, ref, f"stream-K {pattern}", matrix=pattern != "cancel")
    assert dg.poll_device_error() == 0


def test_streamk_repeats_bit_identical(dg, orc):
    case = workloads.dense(64, 7168, 4096, seed=11, a_std=1.0, b_std=0.02)
    first, ws, _ = _run(dg, orc, case, "repeat 0")
    dg.set_kernel_family(5)
    try:
        for i in range(3):
            again = P.out_bits(P.run_dense(dg, case, workspace=ws))
            assert np.array_equal(again, first), f"repeat {i + 1} differs"
    finally:
        dg.set_kernel_family(0)
    assert np.all(_counters(dg, ws, case.M, case.N, case.K) == 0)


def test_streamk_opt_in_and_workspace_checks(dg, orc):
    """Automatic mode ignores a workspace (the stream-K kernel is opt-in); family 5 without a
    workspace, or with one too small, is DG_ERR_WORKSPACE and writes nothing.  All results
    match the oracle."""
    case = workloads.dense(64, 4096, 7168, seed=12, a_std=1.0, b_std=0.02)
    ref = orc.gemm_dense(case.a, case.sa, case.b, case.sb)
    ws = dg.workspace_for(case.M, case.N, case.K)
    got = P.out_bits(P.run_dense(dg, case, workspace=ws))
    assert dg.get_last_launch()["family"] != 5
    P.check(got, ref, "auto with workspace")
    got = P.out_bits(P.run_dense(dg, case))
    assert dg.get_last_launch()["family"] != 5
    P.check(got, ref, "auto without workspace")
    dg.set_kernel_family(5)
    try:
        for w in (None, ws[: ws.numel() // 2]):
            d = P.sentinel_out((case.M, case.N))
            with pytest.raises(dg.DGError) as e:
                P.run_dense(dg, case, d=d, workspace=w)
            assert e.value.status == dg.DG_ERR_WORKSPACE
            assert np.all(P.out_bits(d) == P.SENTINEL)
    finally:
        dg.set_kernel_family(0)
    assert dg.poll_device_error() == 0


def test_streamk_misaligned_workspace_rejected(dg):
    case = workloads.dense(64, 2112, 4096, seed=13)
    ws = dg.workspace_for(case.M, case.N, case.K)
    buf = torch.zeros(ws.numel() + 512, dtype=torch.uint8, device="cuda")
    d = P.sentinel_out((case.M, case.N))
    dg.set_kernel_family(5)
    try:
        with pytest.raises(dg.DGError) as e:
            P.run_dense(dg, case, d=d, workspace=buf[16:16 + ws.numel()])
    finally:
        dg.set_kernel_family(0)
    assert e.value.status == dg.DG_ERR_INVALID_ARG
    assert np.all(P.out_bits(d) == P.SENTINEL)


def test_streamk_fewer_sms(dg, orc):
    """With an SM budget of 37 the partition changes (fewer, longer ranges); the workspace
    size follows the budget."""
    case = workloads.dense(64, 2112, 4096, seed=14, a_std=1.0, b_std=0.02)
    full = dg.get_workspace_size(0, case.M, case.N, case.K)
    prev = dg.set_num_sms(37)
    try:
        assert dg.get_workspace_size(0, case.M, case.N, case.K) < full
        got, _, _ = _run(dg, orc, case, "37 SMs")
        assert dg.get_last_launch()["grid"] == 37
    finally:
        dg.set_num_sms(prev)


def test_streamk_watchdog_then_recovers(dg, orc):
    """The fault-injection hook makes the MMA issuer wait on a barrier nothing signals: the
    kernel gives up after the (1 ms) limit, reports DG_ERR_TIMEOUT and returns; after the
    workspace is zero-filled again the next call matches the oracle."""
    case = workloads.dense(64, 2112, 2048, seed=15, a_std=1.0, b_std=0.02)
    ws = dg.workspace_for(case.M, case.N, case.K)
    prev_t = dg.set_wait_timeout_ns(1_000_000)
    dg.set_fault_injection(1)
    dg.set_kernel_family(5)
    try:
        P.run_dense(dg, case, workspace=ws)
    finally:
        dg.set_fault_injection(0)
        dg.set_kernel_family(0)
        dg.set_wait_timeout_ns(prev_t)
    assert dg.poll_device_error() == dg.DG_ERR_TIMEOUT
    ws.zero_()
    _run(dg, orc, case, "after timeout")
