"""GPU parity of the per-token FP8 quantisation kernel against the oracle: the e4m3 codes and
the fp32 scales must be bit-identical (both sides take every rounding decision in the same
fp32 operations).  Covers ragged M (scale-layout padding), one K block, edge tiles (all zero,
below the 1e-4 floor, a single outlier, exact e4m3 midpoints), a full DeepSeek-sized
activation, and quantise -> GEMM against the oracle GEMM on the oracle's codes."""
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
    return mod


@pytest.fixture(scope="module")
def orc():
    import oracle
    oracle.build()
    return oracle


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _run(dg, bits: np.ndarray):
    M, K = bits.shape
    x = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    m4 = dg.get_tma_aligned_size(M, 4)
    sfa = torch.full((K // 128, m4), -7.0, dtype=torch.float32, device="cuda")  # sentinel
    q, sfa = dg.quantize_fp8_1x128(x, sfa=sfa)
    torch.cuda.synchronize()
    return q.cpu().numpy(), sfa.cpu().numpy()


def _check(dg, orc, bits):
    M, K = bits.shape
    q, sfa = _run(dg, bits)
    rq, rsa = orc.quantize_1x128(bits)
    assert np.array_equal(q, rq), f"{np.count_nonzero(q != rq)} codes differ"
    assert np.array_equal(sfa[:, :M].T.view(np.uint32), rsa.view(np.uint32)), "scales differ"
    assert np.all(sfa[:, M:] == -7.0), "padding of the scale layout was written"


@pytest.mark.parametrize("M,K", [(1, 128), (5, 256), (130, 384), (33, 7168), (1000, 1536)])
def test_quant_parity_random(dg, orc, M, K):
    rng = np.random.default_rng(M * 31 + K)
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    x[rng.random((M, K)) < 0.01] *= 50.0
    _check(dg, orc, _bf16_bits(x))


def test_quant_edge_tiles(dg, orc):
    rng = np.random.default_rng(5)
    M, K = 12, 1024
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    x[0, :128] = 0.0                              # all zero
    x[1, 128:256] = -0.0                          # negative zeros
    x[2, 256:384] *= 1e-7                          # below the 1e-4 floor
    x[3, :] = 1e-3
    x[3, 5] = -3.0e4                               # one outlier per tile row
    x[4, 384:512] = np.float32(2.0 ** -130)        # fp32 subnormals -> bf16 subnormals
    # a tile whose amax is exactly 448, so the factor 448 / amax is exactly 1 and x * factor = x:
    # e4m3 midpoints then exercise the ties-to-even rounding of the kernel's conversion
    mids = [1.0625, 1.1875, 2.125, 0.0078125 * 1.5, 240.0, 416.0, -1.0625, -2.375]
    x[5, 512:640] = 0.5
    x[5, 512] = 448.0
    x[5, 513:513 + len(mids)] = mids
    _check(dg, orc, _bf16_bits(x))


def test_quant_full_size(dg, orc):
    """A DeepSeek-V3-sized activation (4096 tokens x hidden 7168), every code compared."""
    rng = np.random.default_rng(7)
    x = rng.normal(0, 1, (4096, 7168)).astype(np.float32)
    x[rng.random(x.shape) < 0.01] *= 50.0
    _check(dg, orc, _bf16_bits(x))


def test_quant_then_gemm(dg, orc):
    """Quantise on the GPU, multiply on the GPU; compare with the oracle GEMM on the oracle's
    own codes and scales."""
    rng = np.random.default_rng(9)
    M, N, K = 300, 1040, 1536
    bits = _bf16_bits(rng.normal(0, 1, (M, K)).astype(np.float32))
    x = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    q, sfa = dg.quantize_fp8_1x128(x)
    case = workloads.dense(M, N, K, seed=91)
    b = torch.from_numpy(case.b).cuda()
    sfb = torch.from_numpy(case.sb).cuda()
    d = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    dg.dg_gemm_fp8_fp8_bf16_nt(q, sfa, b, sfb, d)
    torch.cuda.synchronize()
    rq, rsa = orc.quantize_1x128(bits)
    ref = orc.gemm_dense(rq, rsa, case.b, case.sb)
    P.assert_close(P.out_bits(d), ref.bits, ref.mag, "quantise -> GEMM", acc=ref.acc)


def test_quant_all_bf16_patterns_awkward_scales(dg, orc):
    """Every finite bf16 bit pattern, in tiles whose amax gives inexact factors 448 / amax:
    every product x * factor and its e4m3 rounding (near midpoints, in the subnormal range,
    at saturation) must match the oracle bit for bit."""
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    exp = (pats >> 7) & 0xFF
    pats = pats[exp != 0xFF]                       # drop inf / NaN
    rng = np.random.default_rng(21)
    amaxes = [0.7, 1.3, 3.14159, 0.0123, 77.7, 1e3, 2.9e4, 5.5e-3, 448.0 / 3.0, 0.999]
    rows = []
    for a in amaxes:
        a_bits = _bf16_bits(np.array([a], np.float32))[0]
        a_val = float(np.array([np.uint32(a_bits) << 16], np.uint32).view(np.float32)[0])
        vals = (np.array(pats, np.uint32) << 16).view(np.float32)
        keep = pats[np.abs(vals) <= a_val]
        keep = keep[rng.permutation(len(keep))]
        n = (len(keep) // 127) * 127
        tiles = keep[:n].reshape(-1, 127)
        col = np.full((tiles.shape[0], 1), a_bits, np.uint16)
        rows.append(np.concatenate([col, tiles], axis=1))
    bits = np.concatenate(rows, axis=0)
    bits = bits[: (bits.shape[0] // 8) * 8].reshape(-1, 8 * 128)  # 8 tiles per row, K = 1024
    _check(dg, orc, bits)
