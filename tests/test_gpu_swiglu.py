"""GPU parity of the SwiGLU + per-token FP8 quantisation kernel against the oracle.  The
kernel's exp is the GPU's fast exponential, so its y can differ from the oracle's (fp64, rounded
once to fp32) by a few fp32 ulps; the comparison is therefore:
  - scales within 2e-6 relative;
  - every code that the oracle's product y * factor does not put within 1e-5 (relative) of an
    e4m3 rounding midpoint decodes to exactly the oracle's value (the unique answer);
  - next to a midpoint either neighbour is a valid rounding, and nothing else is accepted;
  - rows a masked call must not process keep their sentinel codes and scales."""
from __future__ import annotations

import numpy as np
import pytest
import torch

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


def _decode_table(orc):
    return np.array([orc.e4m3_decode(c) for c in range(256)], dtype=np.float64)


def _grid(orc):
    return np.array(sorted({orc.e4m3_decode(c) for c in range(0x7F)}), dtype=np.float64)


def _compare(orc, q, sa, rq, rsa, y, rows):
    """q/sa: kernel codes [M, I] and logical scales [M, I/128]; rq/rsa/y: oracle's."""
    dec = _decode_table(orc)
    grid = _grid(orc)
    q, rq, y = q[rows], rq[rows], y[rows]
    sa, rsa = sa[rows], rsa[rows]
    assert np.allclose(sa, rsa, rtol=2e-6, atol=0), "scales differ"
    M, I = q.shape
    amax = np.maximum(np.abs(y.reshape(M, I // 128, 128)).max(axis=2), np.float32(1e-4)).astype(np.float32)
    factor = (np.float32(448.0) / amax).astype(np.float32)  # the oracle's own per-tile factor
    p = np.abs((y * np.repeat(factor, 128, axis=1)).astype(np.float32).astype(np.float64))
    idx = np.clip(np.searchsorted(grid, p), 1, len(grid) - 1)
    lo, hi = grid[idx - 1], grid[idx]
    mid = (lo + hi) / 2
    near = np.abs(p - mid) <= 1e-5 * np.maximum(p, 1e-30)
    dk, do = dec[q], dec[rq]
    same = dk == do
    assert np.all(same | near), f"{np.count_nonzero(~(same | near))} codes differ away from a midpoint"
    # next to a midpoint: the kernel's value must be one of the two neighbours, with the sign of y
    nb_ok = (np.abs(np.abs(dk) - lo) == 0) | (np.abs(np.abs(dk) - hi) == 0)
    assert np.all(same | (near & nb_ok))
    return int(np.count_nonzero(near & ~same))


def _run(dg, bits, masked_m=None, rows_per_group=0, sentinel=True):
    M = bits.shape[0]
    h = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    I = bits.shape[1] // 2
    q = torch.full((M, I), 0xAA, dtype=torch.uint8, device="cuda")
    mm = None if masked_m is None else torch.tensor(masked_m, dtype=torch.int32, device="cuda")
    if mm is None:
        sfa = torch.full((I // 128, dg.get_tma_aligned_size(M, 4)), -7.0, device="cuda")
    else:
        G = M // rows_per_group
        sfa = torch.full((G, I // 128, dg.get_tma_aligned_size(rows_per_group, 4)), -7.0, device="cuda")
    q, sfa = dg.swiglu_quantize_fp8_1x128(h, mm, rows_per_group, q=q, sfa=sfa)
    torch.cuda.synchronize()
    return q.cpu().numpy(), sfa.cpu().numpy()


@pytest.mark.parametrize("M,I", [(1, 128), (300, 512), (4096, 2048)])
def test_swiglu_parity_dense(dg, orc, M, I):
    rng = np.random.default_rng(M + I)
    x = rng.normal(0, 1.5, (M, 2 * I)).astype(np.float32)
    x[rng.random(x.shape) < 0.005] *= 20.0
    bits = _bf16_bits(x)
    q, sfa = _run(dg, bits)
    rq, rsa, y = orc.swiglu_quantize(bits)
    sa = sfa[:, :M].T
    assert np.all(sfa[:, M:] == -7.0)
    _compare(orc, q, sa, rq, rsa, y, np.arange(M))


def test_swiglu_masked_layout(dg, orc):
    G, R, I = 4, 64, 256
    masked_m = [64, 0, 17, 33]
    rng = np.random.default_rng(11)
    bits = _bf16_bits(rng.normal(0, 2, (G * R, 2 * I)).astype(np.float32))
    q, sfa = _run(dg, bits, masked_m, R)
    valid = np.array([r < masked_m[g] for g in range(G) for r in range(R)])
    rq, rsa, y = orc.swiglu_quantize(bits, row_valid=valid.astype(np.uint8))
    # logical scales of the valid rows from the per-group layout [G][I/128][align4(R)]
    sa = np.zeros((G * R, I // 128), np.float32)
    for g in range(G):
        sa[g * R:(g + 1) * R] = sfa[g, :, :R].T
    _compare(orc, q, sa, rq, rsa, y, np.nonzero(valid)[0])
    assert np.all(q[~valid] == 0xAA), "a row beyond masked_m was written"
    for g in range(G):
        assert np.all(sfa[g, :, masked_m[g]:] == -7.0)


def test_swiglu_then_masked_gemm(dg, orc):
    """The kernel's output feeds the masked grouped GEMM directly (same layouts)."""
    import workloads
    from tests import parity as P
    G, R, I, N = 3, 128, 256, 384
    masked_m = np.array([128, 50, 0], np.int32)
    rng = np.random.default_rng(12)
    bits = _bf16_bits(rng.normal(0, 2, (G * R, 2 * I)).astype(np.float32))
    q, sfa = _run(dg, bits, list(masked_m), R)
    b_case = workloads.masked(G=G, M_max=R, N=N, K=I, seed=13, masked_m=list(masked_m))
    d = torch.full((G, R, N), 0, dtype=torch.bfloat16, device="cuda")
    d.view(torch.int16).fill_(-1)
    dg.dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(
        torch.from_numpy(q).cuda().view(G, R, I), torch.from_numpy(sfa).cuda(),
        torch.from_numpy(b_case.b).cuda(), torch.from_numpy(b_case.sb).cuda(), d,
        torch.from_numpy(masked_m).cuda(), 128)
    torch.cuda.synchronize()
    got = P.out_bits(d)
    # the oracle GEMM on the kernel's own codes and scales
    sa = np.stack([sfa[g, :, :R].T for g in range(G)])
    ref = orc.gemm_masked(q.reshape(G, R, I), sa, b_case.b, b_case.sb, masked_m)
    inv = np.arange(R)[None, :] >= masked_m[:, None]
    assert np.all(got[inv] == P.SENTINEL)
    P.check(got, ref, "swiglu -> masked GEMM", sel=~inv)
