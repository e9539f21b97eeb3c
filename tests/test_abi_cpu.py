"""CPU-side checks of the C ABI: the shared library loads, exports every function that
include/dg.h declares, and rejects bad arguments before touching the device.  No compute call
reaches a GPU here."""
from __future__ import annotations

import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dg.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def dg():
    import __graft_entry__
    __graft_entry__._library_builder().build()
    import fp8_block_scaled_tma_b200 as mod
    return mod


def test_header_declares_the_api():
    names = declared_functions()
    for n in ["dg_gemm_fp8_fp8_bf16_nt", "dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous",
              "dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked", "dg_set_num_sms", "dg_get_num_sms",
              "dg_get_tma_aligned_size", "dg_gemm_fp8_fp4_bf16_nt",
              "dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous",
              "dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked"]:
        assert n in names


def test_library_exports_every_declared_symbol(dg):
    lib = ctypes.CDLL(dg.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in dg.h but not exported"


def test_tma_aligned_size(dg):
    assert dg.get_tma_aligned_size(0, 4) == 0
    assert dg.get_tma_aligned_size(1, 4) == 4
    assert dg.get_tma_aligned_size(4, 4) == 4
    assert dg.get_tma_aligned_size(5, 4) == 8
    assert dg.get_tma_aligned_size(1, 1) == 16
    assert dg.get_tma_aligned_size(17, 2) == 24
    assert dg.get_tma_aligned_size(3, 16) == 3
    assert dg.get_tma_aligned_size(3, 6) == 8       # 8 * 6 = 48
    assert dg.lib.dg_get_tma_aligned_size(-1, 4) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_get_tma_aligned_size(4, 0) == dg.DG_ERR_INVALID_ARG


def test_status_strings(dg):
    for s in range(-6, 1):
        assert dg.status_string(s)
    assert "unknown" in dg.status_string(-99)


def test_num_sms_cap_roundtrip(dg):
    prev = dg.set_num_sms(20)
    assert dg.set_num_sms(0) == 20
    dg.set_num_sms(prev)


def test_config_override_validation(dg):
    assert dg.lib.dg_set_config_override(100, 0, 0) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_set_config_override(0, 1, 0) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_set_config_override(0, 9, 0) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_set_config_override(0, 0, 9) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_set_config_override(96, 4, 3) == dg.DG_OK
    assert dg.lib.dg_set_config_override(0, 0, 0) == dg.DG_OK
    assert dg.lib.dg_set_kernel_family(6) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_set_kernel_family(-1) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_set_kernel_family(5) == 0 and dg.lib.dg_set_kernel_family(4) == 5
    assert dg.lib.dg_set_kernel_family(0) == 4
    assert dg.lib.dg_set_fault_injection(2) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_set_fault_injection(0) == dg.DG_OK
    assert dg.lib.dg_set_kernel_family(0) == dg.DG_OK
    assert dg.lib.dg_set_pdl(2) == dg.DG_ERR_INVALID_ARG
    prev = dg.set_pdl(False)
    assert dg.set_pdl(prev) is False


def test_timeout_setter(dg):
    prev = dg.set_wait_timeout_ns(12345)
    assert dg.set_wait_timeout_ns(0) == 12345
    dg.set_wait_timeout_ns(prev)


FAKE = 0x100000  # 16-byte aligned, never dereferenced by the host code


@pytest.mark.parametrize("M,N,K,ptr_off,expect", [
    (128, 256, 100, 0, -1),      # K % 128 != 0
    (128, 250, 256, 0, -1),      # N % 8 != 0
    (-1, 256, 256, 0, -1),       # negative M
    (128, 256, 256, 4, -1),      # misaligned pointer
    (128, 0, 256, 0, -1),        # N == 0
])
def test_dense_rejects_bad_arguments(dg, M, N, K, ptr_off, expect):
    p = FAKE + ptr_off
    r = dg.lib.dg_gemm_fp8_fp8_bf16_nt(p, FAKE, FAKE, FAKE, FAKE, M, N, K, None, 0, None)
    assert r == expect


def test_null_pointer_rejected(dg):
    assert dg.lib.dg_gemm_fp8_fp8_bf16_nt(None, FAKE, FAKE, FAKE, FAKE, 128, 256, 256, None, 0,
                                          None) == dg.DG_ERR_INVALID_ARG


def test_grouped_reject_bad_arguments(dg):
    L = dg.lib
    # contiguous: M_total not a multiple of 128, G <= 0, null index array
    assert L.dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 100,
                                                          256, 256, 2, None, 0, None) == -1
    assert L.dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128,
                                                          256, 256, 0, None, 0, None) == -1
    assert L.dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(FAKE, FAKE, FAKE, FAKE, FAKE, None, 128,
                                                          256, 256, 2, None, 0, None) == -1
    # masked: G <= 0, negative expected_m, null masked_m
    assert L.dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 256,
                                                      256, 256, 128, None, 0, None) == -1
    assert L.dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 256,
                                                      256, 256, -1, None, 0, None) == -1
    assert L.dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 256,
                                                      256, 256, 128, None, 0, None) == -1


def test_masked_group_limit(dg):
    L = dg.lib
    assert L.dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1025,
                                                      128, 256, 256, 64, None, 0, None) == -1
    assert L.dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1024,
                                                      0, 256, 256, 64, None, 0, None) == 0


def test_fp4_entries_reject_bad_arguments(dg):
    L = dg.lib
    # packed E2M1 B must be 32-byte aligned (16 is enough for e4m3 B)
    assert L.dg_gemm_fp8_fp4_bf16_nt(FAKE, FAKE, FAKE + 16, FAKE, FAKE, 128, 256, 256, None) == -1
    assert L.dg_gemm_fp8_fp4_bf16_nt(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 200, None) == -1
    assert L.dg_gemm_fp8_fp4_bf16_nt(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 256, 256, None) == 0
    assert L.dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous(FAKE, FAKE, FAKE + 16, FAKE, FAKE, FAKE,
                                                          128, 256, 256, 2, None) == -1
    assert L.dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous(FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                                          128, 256, 256, 2, None) == -1
    assert L.dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked(FAKE, FAKE, FAKE + 16, FAKE, FAKE, FAKE, 2,
                                                      128, 256, 256, 64, None) == -1
    assert L.dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0,
                                                      128, 256, 256, 64, None) == -1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_fp4_valid_call_without_device_is_unsupported(dg):
    r = dg.lib.dg_gemm_fp8_fp4_bf16_nt(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 256, None)
    assert r == dg.DG_ERR_UNSUPPORTED


def test_empty_problems_are_noops(dg):
    L = dg.lib
    assert L.dg_gemm_fp8_fp8_bf16_nt(None, None, None, None, None, 0, 256, 256, None, 0, None) == 0
    assert L.dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(None, None, None, None, None, None, 0,
                                                          256, 256, 2, None, 0, None) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_is_unsupported(dg):
    r = dg.lib.dg_gemm_fp8_fp8_bf16_nt(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 256, None, 0, None)
    assert r == dg.DG_ERR_UNSUPPORTED
    assert dg.lib.dg_get_num_sms() == dg.DG_ERR_UNSUPPORTED


def test_sfa_layout_helper(dg):
    sa = torch.arange(6 * 3, dtype=torch.float32).reshape(6, 3)
    mn = dg.sfa_mn_major(sa)
    assert mn.shape == (3, 8)
    assert torch.equal(mn[:, :6], sa.t())
    assert torch.all(mn[:, 6:] == 0)
    sa3 = torch.arange(2 * 5 * 2, dtype=torch.float32).reshape(2, 5, 2)
    mn3 = dg.sfa_mn_major(sa3)
    assert mn3.shape == (2, 2, 8)
    assert torch.equal(mn3[1, :, :5], sa3[1].t())


def test_quantize_rejects_bad_arguments(dg):
    L = dg.lib
    assert L.dg_quantize_fp8_1x128(FAKE, FAKE, FAKE, 4, 100, None) == dg.DG_ERR_INVALID_ARG   # K % 128
    assert L.dg_quantize_fp8_1x128(FAKE, FAKE, FAKE, -1, 128, None) == dg.DG_ERR_INVALID_ARG  # M < 0
    assert L.dg_quantize_fp8_1x128(FAKE + 4, FAKE, FAKE, 4, 128, None) == dg.DG_ERR_INVALID_ARG
    assert L.dg_quantize_fp8_1x128(None, FAKE, FAKE, 4, 128, None) == dg.DG_ERR_INVALID_ARG
    assert L.dg_quantize_fp8_1x128(None, None, None, 0, 128, None) == dg.DG_OK  # empty: no-op


def test_workspace_size_without_a_device(dg):
    """Without a usable device no call can use a workspace: the size is 0 and workspace_for
    gives None (the GEMMs never require one)."""
    if torch.cuda.is_available():
        pytest.skip("checks the no-device answer")
    assert dg.get_workspace_size(0, 64, 7168, 16384) == 0
    assert dg.workspace_for(64, 7168, 16384) is None
    assert dg.get_workspace_size(1, 64, 7168, 16384) == 0
