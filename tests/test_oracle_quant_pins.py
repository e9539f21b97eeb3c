"""Pins of the oracle's per-token FP8 quantisation (the step before the GEMM: one fp32 scale
per 1 x 128 tile of the activations, DeepGEMM release write-up, "深入了解DeepGEMM").  The E4M3
encoder is checked against the format's own grid (every code round-trips, ties go to the even
code) and against torch's independent float8_e4m3fn cast; the quantiser against properties that
any correct implementation has (the largest element maps to +-448, all-zero tiles use the 1e-4
floor, every element is the nearest grid point of x * (448 / amax)) and against a numpy/torch
composition on random data."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle


@pytest.fixture(scope="module", autouse=True)
def _built():
    oracle.build()


FINITE = [c for c in range(256) if c not in (0x7F, 0xFF)]


def test_every_finite_code_round_trips():
    for c in FINITE:
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c, hex(c)


def test_nan_encodes_to_nan_code():
    assert oracle.e4m3_encode(float("nan")) == 0x7F


def test_midpoints_round_to_even_code():
    pos = [c for c in range(0x00, 0x7F)]  # +0 .. 448 in increasing order
    for c in pos[:-1]:
        lo, hi = oracle.e4m3_decode(c), oracle.e4m3_decode(c + 1)
        mid = (lo + hi) / 2  # exact in fp32: both neighbours have <= 4 significant bits
        even = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(mid) == even, (hex(c), mid)
        assert oracle.e4m3_encode(-mid) == 0x80 | even
        # just off the midpoint: the nearer neighbour
        eps = (hi - lo) / 64
        assert oracle.e4m3_encode(mid - eps) == c
        assert oracle.e4m3_encode(mid + eps) == c + 1


def test_saturation():
    for v in (448.0, 448.5, 463.9, 464.0, 1e4, 3.0e38):
        assert oracle.e4m3_encode(v) == 0x7E
        assert oracle.e4m3_encode(-v) == 0xFE


def test_encoder_matches_torch_cast():
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.uniform(-448, 448, 4000),
        rng.normal(0, 1, 4000),
        rng.normal(0, 1e-2, 2000),
        np.ldexp(rng.uniform(-1, 1, 2000), -8),  # subnormal range of e4m3
    ]).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, ref)


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def test_quantise_properties():
    rng = np.random.default_rng(12)
    M, K = 7, 384
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    x[1, :128] = 0.0                      # an all-zero tile
    x[2, 128:256] *= 1e-6                 # a tile below the 1e-4 floor
    x[3, 256] = -1000.0                   # a negative outlier
    bits = _bf16_bits(x)
    xf = _bits_to_f32(bits)
    q, sa = oracle.quantize_1x128(bits)
    assert q.shape == (M, K) and sa.shape == (M, K // 128)
    floor = np.float32(1e-4) / np.float32(448.0)
    assert sa[1, 0] == floor and np.all(q[1, :128] == 0)
    assert sa[2, 1] == floor
    assert q[3, 256] == 0xFE
    for m in range(M):
        for kb in range(K // 128):
            t = xf[m, kb * 128:(kb + 1) * 128]
            amax = np.float32(np.abs(t).max())
            amax_c = np.float32(max(amax, np.float32(1e-4)))
            s = amax_c / np.float32(448.0)
            assert sa[m, kb] == s
            codes = q[m, kb * 128:(kb + 1) * 128]
            if amax >= 1e-4:
                assert np.any((codes & 0x7F) == 0x7E)  # the largest element maps to +-448
            # each code is the nearest grid point of x * (448 / amax) (ties to even)
            quot = (t * (np.float32(448.0) / amax_c)).astype(np.float32)
            dec = np.array([oracle.e4m3_decode(int(c)) for c in codes])
            for v, d in zip(quot, dec):
                v = float(v)
                if abs(v) >= 448.0:
                    assert abs(d) == 448.0
                    continue
                err = abs(d - v)
                nb = [oracle.e4m3_decode(c) for c in FINITE]
                assert err <= min(abs(n - v) for n in nb) + 0.0


def test_quantise_matches_numpy_torch_composition():
    rng = np.random.default_rng(13)
    M, K = 64, 1024
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    x[rng.random((M, K)) < 0.01] *= 50.0
    bits = _bf16_bits(x)
    xf = _bits_to_f32(bits).reshape(M, K // 128, 128)
    amax = np.maximum(np.abs(xf).max(axis=2), np.float32(1e-4)).astype(np.float32)
    s = amax / np.float32(448.0)
    factor = np.float32(448.0) / amax
    quot = (xf * factor[:, :, None]).astype(np.float32).reshape(M, K)
    ref_q = torch.from_numpy(np.clip(quot, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    q, sa = oracle.quantize_1x128(bits)
    assert np.array_equal(sa, s)
    assert np.array_equal(q, ref_q)


def test_quantise_departs_from_the_division_form_only_next_to_midpoints():
    """Bounds the oracle's quantiser against the plain definition of the quantisation,
    code = e4m3(x / scale) with scale = amax / 448 -- the form the GEMM harness uses for its
    synthetic inputs, here evaluated as one fp32 division and cast by torch's independent
    float8_e4m3fn conversion.  The oracle multiplies by the fp32 factor 448 / amax instead.  Both
    quotients lie within 2^-24 relative (one fp32 rounding each, plus the rounding of the factor
    or of the scale) of the exact x / scale, so where the two codes differ an E4M3 rounding
    midpoint must lie within a few 2^-24 of it, and the codes must be neighbours (same sign,
    magnitudes one code apart).  Everywhere else the codes are equal."""
    rng = np.random.default_rng(14)
    M, K = 2048, 1024
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    x[rng.random((M, K)) < 0.01] *= 50.0
    x[: M // 4] = rng.uniform(-3.0, 3.0, (M // 4, K)).astype(np.float32)
    x[M // 4: M // 2] *= np.float32(1e-3)          # tiles reaching the subnormal codes
    bits = _bf16_bits(x)
    xf = _bits_to_f32(bits)
    q, sa = oracle.quantize_1x128(bits)
    s_full = np.repeat(sa, 128, axis=1)
    div32 = (xf / s_full).astype(np.float32)
    q_div = torch.from_numpy(np.clip(div32, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # the exact quotient (fp64 holds x / scale of two fp32 numbers to 2^-53) and its distance to
    # the nearest rounding midpoint of the E4M3 grid, relative to the quotient
    v = np.abs(xf.astype(np.float64) / s_full.astype(np.float64))
    grid = np.array([oracle.e4m3_decode(c) for c in range(0x7F)])      # +0 .. 448, ascending
    mids = (grid[:-1] + grid[1:]) / 2
    pos = np.clip(np.searchsorted(mids, v), 1, mids.size - 1)
    near = np.minimum(np.abs(v - mids[pos - 1]), np.abs(v - mids[pos]))
    rel = np.where(v > 0, near / np.maximum(v, 1e-300), np.inf)
    differ = q != q_div
    n_near = int(np.count_nonzero(rel < 2.0 ** -21))
    assert n_near > 0, "the sample reached no midpoint: the bound below would be untested"
    assert np.all(rel[differ] < 2.0 ** -21), "codes differ away from a midpoint"
    same_sign = (q[differ] & 0x80) == (q_div[differ] & 0x80)
    step = np.abs((q[differ] & 0x7F).astype(int) - (q_div[differ] & 0x7F).astype(int))
    assert np.all(same_sign) and np.all(step == 1), "differing codes are not neighbours"
    assert np.count_nonzero(differ) <= n_near
    # the scales are the plain definition amax / 448 (floored), bit for bit
    amax = np.maximum(np.abs(xf.reshape(M, K // 128, 128)).max(axis=2), np.float32(1e-4))
    assert np.array_equal(sa, (amax / np.float32(448.0)).astype(np.float32))
