"""Pins of the oracle's SwiGLU + per-token FP8 quantisation (the step between the two grouped
GEMMs of an MoE layer): closed-form SiLU values, agreement of y with torch's fp64 SiLU to one
fp32 rounding, the quantisation of y matching an independent numpy/torch composition, sign
symmetry in the up half, and skipped rows left untouched."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle


@pytest.fixture(scope="module", autouse=True)
def _built():
    oracle.build()


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def test_closed_forms():
    I = 128
    g = np.zeros((1, I), np.float32)
    u = np.ones((1, I), np.float32)
    g[0, :6] = [0.0, 1.0, -1.0, 20.0, -20.0, 2.0]
    u[0, 5] = 0.0
    h = _bf16_bits(np.concatenate([g, u], axis=1))
    _, _, y = oracle.swiglu_quantize(h)
    expect = [0.0, 1 / (1 + math.exp(-1)), -1 / (1 + math.exp(1)), 20 / (1 + math.exp(-20)),
              -20 / (1 + math.exp(20)), 0.0]
    for i, e in enumerate(expect):
        assert y[0, i] == np.float32(e), (i, y[0, i], e)


def test_y_matches_torch_silu():
    rng = np.random.default_rng(3)
    M, I = 16, 256
    h = _bf16_bits(rng.normal(0, 2, (M, 2 * I)))
    _, _, y = oracle.swiglu_quantize(h)
    hf = torch.from_numpy(_f32(h)).double()
    ref = (torch.nn.functional.silu(hf[:, :I]) * hf[:, I:]).float().numpy()
    # the two fp64 formulas round to the same fp32 value except in rare ties: 1 ulp at most
    ulp = np.spacing(np.abs(ref).astype(np.float32))
    assert np.all(np.abs(y - ref) <= ulp)
    assert np.mean(y == ref) > 0.99


def test_quantisation_of_y_matches_numpy_torch():
    rng = np.random.default_rng(4)
    M, I = 32, 512
    x = rng.normal(0, 1, (M, 2 * I)).astype(np.float32)
    x[rng.random(x.shape) < 0.01] *= 30.0
    h = _bf16_bits(x)
    q, sa, y = oracle.swiglu_quantize(h)
    yt = y.reshape(M, I // 128, 128)
    amax = np.maximum(np.abs(yt).max(axis=2), np.float32(1e-4)).astype(np.float32)
    factor = np.float32(448.0) / amax
    prod = (yt * factor[:, :, None]).astype(np.float32).reshape(M, I)
    ref_q = torch.from_numpy(np.clip(prod, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(sa, amax / np.float32(448.0))
    assert np.array_equal(q, ref_q)


def test_sign_symmetry_in_up_half():
    rng = np.random.default_rng(5)
    M, I = 4, 256
    x = rng.normal(0, 1, (M, 2 * I)).astype(np.float32)
    h = _bf16_bits(x)
    h_neg = h.copy()
    h_neg[:, I:] ^= 0x8000  # negate the up half
    q, sa, _ = oracle.swiglu_quantize(h)
    qn, san, _ = oracle.swiglu_quantize(h_neg)
    assert np.array_equal(sa, san)
    nz = (q & 0x7F) != 0
    assert np.array_equal(qn[nz], q[nz] ^ 0x80)


def test_skipped_rows_untouched():
    rng = np.random.default_rng(6)
    M, I = 6, 128
    h = _bf16_bits(rng.normal(0, 1, (M, 2 * I)))
    valid = np.array([1, 0, 1, 1, 0, 1], np.uint8)
    q, sa, y = oracle.swiglu_quantize(h, row_valid=valid)
    qa, saa, _ = oracle.swiglu_quantize(h)
    assert np.all(q[valid == 0] == 0) and np.all(np.isnan(y[valid == 0]))
    assert np.array_equal(q[valid == 1], qa[valid == 1])
    assert np.array_equal(sa[valid == 1], saa[valid == 1])
