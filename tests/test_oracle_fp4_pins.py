"""Pins of the oracle's FP4 (E2M1) operand path of the FP8 x FP4 GEMM (the mixed-precision
variant that the DeepGEMM update news item lists): the E2M1 value table that the OCP format
definition fixes, the exactness of its expansion into E4M3 codes, the nibble order of the packed
layout, and a small FP8 x FP4 GEMM checked in exact rational arithmetic."""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest

import oracle

# OCP microscaling formats, FP4 E2M1: the 8 magnitudes of codes 0..7, then their negatives
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


@pytest.fixture(scope="module", autouse=True)
def _built():
    oracle.build()


def test_e2m1_value_table():
    for c in range(8):
        assert oracle.e2m1_decode(c) == E2M1_TABLE[c]
        assert oracle.e2m1_decode(c | 8) == -E2M1_TABLE[c]
    assert str(oracle.e2m1_decode(8)) == "-0.0"


def test_expansion_into_e4m3_is_exact():
    for c in range(16):
        packed = np.array([[c | (c << 4)]], np.uint8)
        codes = oracle.e2m1_to_e4m3(packed)
        for code in codes[0]:
            assert oracle.e4m3_decode(int(code)) == oracle.e2m1_decode(c)


def test_nibble_order():
    # element 2j is the low nibble of byte j, element 2j + 1 the high nibble
    packed = np.array([[0x21, 0xF7, 0x0A, 0x90]], np.uint8)
    vals = [oracle.e4m3_decode(int(c)) for c in oracle.e2m1_to_e4m3(packed)[0]]
    # 0x21 -> 0.5, 1.0; 0xF7 -> 6.0, -6.0; 0x0A -> -1.0, 0.0; 0x90 -> 0.0, -0.5
    assert vals == [0.5, 1.0, 6.0, -6.0, -1.0, 0.0, 0.0, -0.5]


def test_fp8_fp4_gemm_exact_rationals():
    rng = np.random.default_rng(31)
    M, N, K = 3, 5, 256
    a = rng.integers(0, 256, (M, K), dtype=np.uint8)
    a[(a & 0x7F) == 0x7F] = 0x38                          # no NaN codes
    b_packed = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = rng.uniform(0.5, 2.0, (M, K // 128)).astype(np.float32)
    sb = rng.uniform(0.5, 2.0, (1, K // 128)).astype(np.float32)
    b = oracle.e2m1_to_e4m3(b_packed)
    res = oracle.gemm_dense(a, sa, b, sb)
    for m in range(M):
        for n in range(N):
            exact = Fraction(0)
            for kb in range(K // 128):
                s = Fraction(0)
                for k in range(kb * 128, kb * 128 + 128):
                    byte = int(b_packed[n, k // 2])
                    nib = (byte >> 4) if (k & 1) else (byte & 0xF)
                    s += Fraction(oracle.e4m3_decode(int(a[m, k]))) * Fraction(oracle.e2m1_decode(nib))
                exact += Fraction(float(sa[m, kb])) * Fraction(float(sb[0, kb])) * s
            assert abs(Fraction(float(res.acc[m, n])) - exact) <= Fraction(1, 10 ** 9) * (abs(exact) + 1)


def test_grouped_expansion_is_per_group():
    """The grouped FP8 x FP4 layouts pass B as [G, N, K/2]: the expansion of the whole array
    equals the expansion of each group, and each code decodes to the nibble's E2M1 value."""
    rng = np.random.default_rng(32)
    G, N, K = 3, 5, 256
    packed = rng.integers(0, 256, (G, N, K // 2), dtype=np.uint8)
    whole = oracle.e2m1_to_e4m3(packed)
    assert whole.shape == (G, N, K)
    for g in range(G):
        assert np.array_equal(whole[g], oracle.e2m1_to_e4m3(packed[g]))
    g, n, k = 2, 4, 201
    nib = (int(packed[g, n, k // 2]) >> 4) if (k & 1) else (int(packed[g, n, k // 2]) & 0xF)
    assert oracle.e4m3_decode(int(whole[g, n, k])) == oracle.e2m1_decode(nib)


def test_fp4_masked_gemm_equals_dense_per_group():
    """A masked FP8 x FP4 GEMM computes, for each group, the dense GEMM of its valid rows."""
    rng = np.random.default_rng(33)
    G, M_max, N, K = 2, 4, 8, 256
    a = rng.integers(0, 0x7E, (G, M_max, K), dtype=np.uint8)
    sa = rng.uniform(0.5, 2.0, (G, M_max, K // 128)).astype(np.float32)
    b = oracle.e2m1_to_e4m3(rng.integers(0, 256, (G, N, K // 2), dtype=np.uint8))
    sb = rng.uniform(0.5, 2.0, (G, 1, K // 128)).astype(np.float32)
    masked_m = np.array([3, 0], np.int32)
    res = oracle.gemm_masked(a, sa, b, sb, masked_m)
    dense = oracle.gemm_dense(a[0, :3], sa[0, :3], b[0], sb[0])
    assert np.array_equal(res.bits[0, :3], dense.bits)
    assert np.all(res.bits[0, 3:] == 0xFFFF) and np.all(res.bits[1] == 0xFFFF)
