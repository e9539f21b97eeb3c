"""Pins for the CPU oracle: each test checks the oracle against something other than itself --
the e4m3 format definition and torch's float8 decoder, exact rational arithmetic, numpy's fp64
matmul, closed forms, and special cases that reduce to the dense product.  A plausible slip in
the oracle (a dropped scale, a wrong K-block or N-block index, a transposed operand, a group
mix-up, double rounding to bf16) fails at least one of them.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---- helpers that do not use the oracle -------------------------------------------------

def torch_e4m3_values() -> np.ndarray:
    """Value of every e4m3 code according to torch's float8_e4m3fn -> float32 conversion."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).float().double().numpy()


def bf16_bits_to_float(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def dequant(codes: np.ndarray, scales: np.ndarray, rows_per_scale: int) -> np.ndarray:
    """Real values code*scale for a [R, K] code matrix; scales indexed [r // rows_per_scale,
    k // 128]."""
    lut = torch_e4m3_values()
    v = lut[codes.astype(np.int64)]
    R, K = codes.shape
    s = np.repeat(np.repeat(scales.astype(np.float64), rows_per_scale, axis=0)[:R], 128, axis=1)
    return v * s


def random_codes(rng, shape) -> np.ndarray:
    """Uniform random e4m3 codes with the two NaN codes excluded."""
    c = rng.integers(0, 256, size=shape, dtype=np.int64)
    c = np.where((c & 0x7F) == 0x7F, c - 1, c)
    return c.astype(np.uint8)


def nearest_bf16_is(bits: int, exact) -> bool:
    """True if the bf16 pattern ``bits`` is a nearest bf16 value to ``exact`` (a Fraction or
    float), checked against both neighbours in the same sign."""
    val = Fraction(float(bf16_bits_to_float([bits])[0]))
    exact = Fraction(exact)
    err = abs(val - exact)
    mag = bits & 0x7FFF
    for nb in (mag - 1, mag + 1):
        if 0 <= nb < 0x7F80:
            nv = Fraction(float(bf16_bits_to_float([(bits & 0x8000) | nb])[0]))
            if abs(nv - exact) < err:
                return False
    if mag == 0 and exact != 0:
        # the nearest could have the other sign only if exact rounds to zero: fine
        return abs(exact) <= Fraction(2) ** -134
    return True


# ---- e4m3 decode --------------------------------------------------------------------------

def test_e4m3_decode_matches_torch_for_all_codes(oracle_mod):
    ref = torch_e4m3_values()
    got = np.array([oracle_mod.e4m3_decode(c) for c in range(256)])
    nan_ref, nan_got = np.isnan(ref), np.isnan(got)
    assert np.array_equal(nan_ref, nan_got)
    assert np.array_equal(ref[~nan_ref], got[~nan_got])
    # signed zero
    assert math.copysign(1.0, oracle_mod.e4m3_decode(0x80)) == -1.0
    assert nan_got.sum() == 2 and nan_got[0x7F] and nan_got[0xFF]


def test_e4m3_decode_golden_values(oracle_mod):
    with open(os.path.join(GOLDEN, "e4m3_special_values.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(rows) >= 10
    for code, val in rows:
        got = oracle_mod.e4m3_decode(int(code, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


# ---- bf16 rounding ------------------------------------------------------------------------

def test_bf16_rne_matches_torch_on_fp32_values(oracle_mod):
    # torch rounds fp32 -> bf16 once (nearest-even); on fp32-representable inputs a single
    # fp64 -> bf16 rounding must agree with it bit for bit.
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(3000) * 10.0 ** rng.integers(-40, 38, 3000),
        rng.standard_normal(500) * 1e-39,      # fp32/bf16 subnormals
        (rng.integers(0, 1 << 16, 500).astype(np.uint32) << 16 | 0x8000).view(np.float32),  # exact ties
    ]).astype(np.float32)
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle_mod.bf16_rne(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(ref, got)


@pytest.mark.parametrize("x,bits", [
    (1.0, 0x3F80),
    (1.0 + 2.0 ** -8, 0x3F80),                 # tie -> even (down)
    (1.0 + 3 * 2.0 ** -8, 0x3F82),             # tie -> even (up)
    (1.0 + 2.0 ** -8 + 2.0 ** -40, 0x3F81),    # just above a tie: a double rounding via fp32 gives 0x3F80
    (-(1.0 + 2.0 ** -8 + 2.0 ** -40), 0xBF81),
    (2.0 ** -133, 0x0001),                     # smallest subnormal
    (2.0 ** -134, 0x0000),                     # tie between 0 and 2^-133 -> even
    (3 * 2.0 ** -135, 0x0001),
    (2.0 ** -126, 0x0080),                     # smallest normal
    ((2.0 - 2.0 ** -7) * 2.0 ** 127, 0x7F7F),  # largest finite
    ((2.0 - 2.0 ** -8) * 2.0 ** 127, 0x7F80),  # tie above the largest finite -> even = inf
    (2.0 ** 130, 0x7F80),
    (0.0, 0x0000),
    (-0.0, 0x8000),
])
def test_bf16_rne_closed_forms(oracle_mod, x, bits):
    assert oracle_mod.bf16_rne(x) == bits


# ---- dense GEMM ------------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K,seed", [(1, 1, 128, 0), (3, 2, 256, 1), (2, 3, 384, 2), (5, 4, 128, 3)])
def test_dense_brute_force_exact_rationals(oracle_mod, M, N, K, seed):
    """Tiny cases computed exactly with Python Fractions from torch's e4m3 decoding."""
    rng = np.random.default_rng(seed)
    a = random_codes(rng, (M, K))
    b = random_codes(rng, (N, K))
    sa = (rng.random((M, K // 128)) * 4 + 0.01).astype(np.float32)
    sb = (rng.random((-(-N // 128), K // 128)) * 4 + 0.01).astype(np.float32)
    lut = torch_e4m3_values()
    res = oracle_mod.gemm_dense(a, sa, b, sb)
    for m in range(M):
        for n in range(N):
            exact = Fraction(0)
            for k in range(K):
                exact += (Fraction(lut[a[m, k]]) * Fraction(float(sa[m, k // 128]))
                          * Fraction(lut[b[n, k]]) * Fraction(float(sb[n // 128, k // 128])))
            assert abs(Fraction(res.acc[m, n]) - exact) <= abs(exact) * Fraction(1, 10 ** 14) + Fraction(1, 10 ** 300)
            assert nearest_bf16_is(int(res.bits[m, n]), exact)


def test_dense_vs_numpy_matmul(oracle_mod):
    """Dequantised product through numpy's fp64 matmul; tail N block of 64 rows included."""
    rng = np.random.default_rng(11)
    M, N, K = 7, 192, 512
    a = random_codes(rng, (M, K))
    b = random_codes(rng, (N, K))
    sa = (rng.random((M, K // 128)) + 0.5).astype(np.float32)
    sb = (rng.random((2, K // 128)) + 0.5).astype(np.float32)
    A = dequant(a, sa, 1)
    B = dequant(b, sb, 128)
    ref = A @ B.T
    mag = np.abs(A) @ np.abs(B).T
    res = oracle_mod.gemm_dense(a, sa, b, sb)
    assert np.all(np.abs(res.acc - ref) <= 1e-12 * mag + 1e-300)
    assert np.allclose(res.mag, mag, rtol=1e-12, atol=0)
    # rounding: every output is a nearest bf16 of the fp64 product
    for m in range(M):
        for n in range(0, N, 17):
            assert nearest_bf16_is(int(res.bits[m, n]), float(ref[m, n]))


def test_transposed_operand_detected(oracle_mod):
    """B is [N, K] (the transposed right-hand side): swapping the roles must change the result."""
    rng = np.random.default_rng(5)
    K = 256
    a = random_codes(rng, (4, K))
    b = random_codes(rng, (4, K))
    sa = np.ones((4, 2), np.float32)
    sb = np.ones((1, 2), np.float32)
    r1 = oracle_mod.gemm_dense(a, sa, b, sb)
    r2 = oracle_mod.gemm_dense(b, sa, a, sb)
    ref = dequant(a, sa, 1) @ dequant(b, sb, 128).T
    assert np.allclose(r1.acc, ref, rtol=1e-13, atol=0)
    assert np.allclose(r2.acc, ref.T, rtol=1e-13, atol=0)


def test_identity_b_closed_form(oracle_mod):
    """B = I (code 0x38 = 1.0 on the diagonal), sb = 1, power-of-two sa: D = a * sa exactly."""
    rng = np.random.default_rng(3)
    M, K = 9, 256
    N = K
    a = random_codes(rng, (M, K))
    sa = (2.0 ** rng.integers(-3, 4, (M, K // 128))).astype(np.float32)
    b = np.zeros((N, K), np.uint8)
    b[np.arange(N), np.arange(N)] = 0x38
    sb = np.ones((2, 2), np.float32)
    res = oracle_mod.gemm_dense(a, sa, b, sb)
    lut = torch_e4m3_values()
    expect = lut[a] * np.repeat(sa.astype(np.float64), 128, axis=1)
    assert np.array_equal(bf16_bits_to_float(res.bits), expect)
    assert np.array_equal(res.acc, expect)


@pytest.mark.parametrize("Kb,q", [(1, 0), (4, -3), (8, 5)])
def test_all_ones_power_of_two_scales(oracle_mod, Kb, q):
    """A = B = 1 (code 0x38), sa[m][kb] = 2^kb, sb = 2^q: D = 128 * 2^q * (2^Kb - 1)."""
    M, N, K = 3, 130, 128 * Kb
    a = np.full((M, K), 0x38, np.uint8)
    b = np.full((N, K), 0x38, np.uint8)
    sa = np.tile((2.0 ** np.arange(Kb)).astype(np.float32), (M, 1))
    sb = np.full((2, Kb), 2.0 ** q, np.float32)
    res = oracle_mod.gemm_dense(a, sa, b, sb)
    expect = 128.0 * 2.0 ** q * (2.0 ** Kb - 1)
    assert np.all(res.acc == expect)
    assert np.all(bf16_bits_to_float(res.bits) == expect)


def test_n_block_indexing_with_tail(oracle_mod):
    """N = 2112 (16 full blocks + a 64-row tail).  A = B = 1, sa = (1, 4) over the two K
    blocks, sb[nb] = (2^(nb-8), 2^(nb-7)): D[m, n] = 128 * 2^(nb-8) * (1 + 8) with
    nb = n // 128.  A swapped K-block pairing gives 6 instead of 9; a wrong N block gives a
    different power of two."""
    M, N, K = 2, 2112, 256
    a = np.full((M, K), 0x38, np.uint8)
    b = np.full((N, K), 0x38, np.uint8)
    sa = np.tile(np.array([1.0, 4.0], np.float32), (M, 1))
    nb = np.arange(17)
    sb = np.stack([2.0 ** (nb - 8), 2.0 ** (nb - 7)], axis=1).astype(np.float32)
    res = oracle_mod.gemm_dense(a, sa, b, sb)
    expect = 128.0 * 9.0 * 2.0 ** (np.arange(N) // 128 - 8)
    assert np.array_equal(res.acc, np.tile(expect, (M, 1)))
    assert np.array_equal(bf16_bits_to_float(res.bits), np.tile(expect, (M, 1)))


def test_cancellation_inside_one_slice_is_exact(oracle_mod):
    """448*448 - 448*448 + 2^-9 * 2^-9 inside one 128-K slice: the slice sum is exactly 2^-18."""
    K = 128
    a = np.zeros((1, K), np.uint8)
    b = np.zeros((1, K), np.uint8)
    a[0, :3] = [0x7E, 0xFE, 0x01]
    b[0, :3] = [0x7E, 0x7E, 0x01]
    res = oracle_mod.gemm_dense(a, np.ones((1, 1), np.float32), b, np.ones((1, 1), np.float32))
    assert res.acc[0, 0] == 2.0 ** -18
    assert res.mag[0, 0] == 2 * 448.0 ** 2 + 2.0 ** -18


def test_row_subset_matches_full(oracle_mod):
    rng = np.random.default_rng(9)
    a = random_codes(rng, (6, 256))
    b = random_codes(rng, (20, 256))
    sa = rng.random((6, 2)).astype(np.float32)
    sb = rng.random((1, 2)).astype(np.float32)
    full = oracle_mod.gemm_dense(a, sa, b, sb)
    part = oracle_mod.gemm_dense(a, sa, b, sb, rows=[5, 0, 3])
    assert np.array_equal(part.bits, full.bits[[5, 0, 3]])


def test_bad_arguments_rejected(oracle_mod):
    a = np.zeros((2, 100), np.uint8)
    with pytest.raises(ValueError):
        oracle_mod.gemm_dense(a, np.ones((2, 1), np.float32), a, np.ones((1, 1), np.float32))


# ---- grouped GEMMs ----------------------------------------------------------------------------

def _grouped_inputs(rng, G, rows, N, K):
    a = random_codes(rng, (rows, K))
    sa = (rng.random((rows, K // 128)) + 0.25).astype(np.float32)
    b = random_codes(rng, (G, N, K))
    sb = (rng.random((G, -(-N // 128), K // 128)) + 0.25).astype(np.float32)
    return a, sa, b, sb


def test_contiguous_rows_use_their_expert(oracle_mod):
    """Each valid row equals the dense product with its own expert's B and sb; -1 rows keep
    the fill pattern bit for bit."""
    rng = np.random.default_rng(21)
    G, N, K = 3, 136, 256
    m_idx = np.array([0, 0, 2, -1, 1, 1, -1, 2, 0, -1], np.int32)
    a, sa, b, sb = _grouped_inputs(rng, G, len(m_idx), N, K)
    res = oracle_mod.gemm_contiguous(a, sa, b, sb, m_idx, out_fill=0xFFFF)
    for r, g in enumerate(m_idx):
        if g < 0:
            assert np.all(res.bits[r] == 0xFFFF) and np.all(np.isnan(res.acc[r]))
        else:
            ref = dequant(a[r:r + 1], sa[r:r + 1], 1) @ dequant(b[g], sb[g], 128).T
            d = oracle_mod.gemm_dense(a[r:r + 1], sa[r:r + 1], b[g], sb[g])
            assert np.array_equal(res.bits[r], d.bits[0])
            assert np.all(np.abs(res.acc[r] - ref[0]) <= 1e-12 * res.mag[r])


def test_contiguous_single_group_equals_dense(oracle_mod):
    rng = np.random.default_rng(22)
    a, sa, b, sb = _grouped_inputs(rng, 1, 12, 64, 384)
    res = oracle_mod.gemm_contiguous(a, sa, b, sb, np.zeros(12, np.int32))
    d = oracle_mod.gemm_dense(a, sa, b[0], sb[0])
    assert np.array_equal(res.bits, d.bits)


def test_contiguous_bad_index_rejected(oracle_mod):
    rng = np.random.default_rng(23)
    a, sa, b, sb = _grouped_inputs(rng, 2, 4, 16, 128)
    with pytest.raises(ValueError):
        oracle_mod.gemm_contiguous(a, sa, b, sb, np.array([0, 1, 2, -1], np.int32))


@pytest.mark.parametrize("masked_m", [[0, 0], [1, 256], [127, 128], [129, 0], [256, 256]])
def test_masked_rows(oracle_mod, masked_m):
    """Rows below masked_m[g] equal the dense product of that group; the rest keep the fill."""
    rng = np.random.default_rng(31)
    G, M_max, N, K = 2, 256, 24, 128
    a, sa, b, sb = _grouped_inputs(rng, G, G * M_max, N, K)
    a3 = a.reshape(G, M_max, K)
    sa3 = sa.reshape(G, M_max, 1)
    res = oracle_mod.gemm_masked(a3, sa3, b, sb, np.array(masked_m, np.int32), out_fill=0xABCD)
    for g in range(G):
        mm = masked_m[g]
        assert np.all(res.bits[g, mm:] == 0xABCD)
        if mm:
            d = oracle_mod.gemm_dense(a3[g, :mm], sa3[g, :mm], b[g], sb[g])
            assert np.array_equal(res.bits[g, :mm], d.bits)
            ref = dequant(a3[g, :mm], sa3[g, :mm], 1) @ dequant(b[g], sb[g], 128).T
            assert np.all(np.abs(res.acc[g, :mm] - ref) <= 1e-12 * res.mag[g, :mm])


def test_masked_bad_count_rejected(oracle_mod):
    rng = np.random.default_rng(32)
    a, sa, b, sb = _grouped_inputs(rng, 1, 4, 16, 128)
    with pytest.raises(ValueError):
        oracle_mod.gemm_masked(a.reshape(1, 4, 128), sa.reshape(1, 4, 1), b, sb,
                               np.array([5], np.int32))
