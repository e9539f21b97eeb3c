"""Seeded synthetic inputs for the FP8 block-scaled GEMM, shared by the tests, the smoke check
and the benchmark.

This module holds no arithmetic of the GEMM itself.  It draws fp32 matrices from a seeded
CPU generator and turns them into the inputs the method consumes: e4m3 codes plus one fp32
scale per 1x128 tile of A and per 128x128 block of B (the DeepSeek-V3 fine-grained scaling
that the DeepGEMM write-up names in "深入了解DeepGEMM").  The scale of a tile is its
absolute maximum divided by 448 (the largest finite e4m3 magnitude), clamped away from zero;
the code is the tile divided by its scale, cast to e4m3 with round-to-nearest-even by torch.
Both the oracle and the CUDA library consume the same codes and scales, so this step does not
enter the parity comparison.

Every array returned here is a CPU numpy/torch array in the LOGICAL layout:
  a codes [rows, K] uint8, sa [rows, K/128] float32,
  b codes [N, K] uint8 (grouped: [G, N, K]), sb [ceil(N/128), K/128] (grouped: [G, ...]).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK = 128
E4M3_MAX = 448.0
AMAX_FLOOR = 1e-4


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def quantise_rows_1x128(x: torch.Tensor):
    """fp32 [R, K] -> (codes uint8 [R, K], scales fp32 [R, K/128]); one scale per 1x128 tile."""
    R, K = x.shape
    assert K % BLOCK == 0
    t = x.float().reshape(R, K // BLOCK, BLOCK)
    amax = t.abs().amax(dim=2).clamp_min(AMAX_FLOOR)
    scale = (amax / E4M3_MAX).float()
    codes = (t / scale.unsqueeze(2)).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.reshape(R, K).numpy(), scale.numpy()


def quantise_blocks_128x128(x: torch.Tensor):
    """fp32 [N, K] -> (codes uint8 [N, K], scales fp32 [ceil(N/128), K/128]); one scale per
    128x128 block (a partial last block of rows gets its own scale over its real rows)."""
    N, K = x.shape
    assert K % BLOCK == 0
    Nb, Kb = -(-N // BLOCK), K // BLOCK
    pad = Nb * BLOCK - N
    xp = torch.nn.functional.pad(x.float(), (0, 0, 0, pad)) if pad else x.float()
    t = xp.reshape(Nb, BLOCK, Kb, BLOCK)
    amax = t.abs().amax(dim=(1, 3)).clamp_min(AMAX_FLOOR)
    scale = (amax / E4M3_MAX).float()
    q = (t / scale[:, None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    codes = q.reshape(Nb * BLOCK, K)[:N]
    return codes.contiguous().numpy(), scale.numpy()


@dataclass
class Dense:
    M: int
    N: int
    K: int
    a: np.ndarray
    sa: np.ndarray
    b: np.ndarray
    sb: np.ndarray

    @property
    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K


@dataclass
class Contiguous:
    G: int
    N: int
    K: int
    counts: np.ndarray          # valid rows per expert
    m_indices: np.ndarray       # int32 [M_total], expert or -1
    a: np.ndarray               # [M_total, K]
    sa: np.ndarray              # [M_total, K/128]
    b: np.ndarray               # [G, N, K]
    sb: np.ndarray              # [G, ceil(N/128), K/128]

    @property
    def M_total(self) -> int:
        return int(self.a.shape[0])

    @property
    def flops(self) -> float:
        return 2.0 * float(self.counts.sum()) * self.N * self.K


@dataclass
class Masked:
    G: int
    M_max: int
    N: int
    K: int
    expected_m: int
    masked_m: np.ndarray        # int32 [G]
    a: np.ndarray               # [G, M_max, K]
    sa: np.ndarray              # [G, M_max, K/128]
    b: np.ndarray               # [G, N, K]
    sb: np.ndarray              # [G, ceil(N/128), K/128]

    @property
    def flops(self) -> float:
        return 2.0 * float(self.masked_m.sum()) * self.N * self.K


def dense(M: int, N: int, K: int, seed: int, a_std: float = 1.0, b_std: float = 1.0,
          outlier_frac: float = 0.0, outlier_scale: float = 50.0) -> Dense:
    """A ~ N(0, a_std^2) [M,K], B ~ N(0, b_std^2) [N,K]; draw order A, B, then (if
    outlier_frac > 0) an independent Bernoulli(outlier_frac) mask over A whose elements are
    multiplied by outlier_scale before quantisation."""
    g = _gen(seed)
    A = torch.randn(M, K, generator=g) * a_std
    B = torch.randn(N, K, generator=g) * b_std
    if outlier_frac > 0:
        mask = torch.rand(M, K, generator=g) < outlier_frac
        A = torch.where(mask, A * outlier_scale, A)
    a, sa = quantise_rows_1x128(A)
    b, sb = quantise_blocks_128x128(B)
    return Dense(M, N, K, a, sa, b, sb)


def _grouped_b(G: int, N: int, K: int, std: float, g: torch.Generator):
    Nb, Kb = -(-N // BLOCK), K // BLOCK
    b = np.empty((G, N, K), np.uint8)
    sb = np.empty((G, Nb, Kb), np.float32)
    for e in range(G):
        be, se = quantise_blocks_128x128(torch.randn(N, K, generator=g) * std)
        b[e], sb[e] = be, se
    return b, sb


def contiguous(G: int, N: int, K: int, seed: int, count_lo: int = 128, count_hi: int = 1024,
               a_std: float = 1.0, b_std: float = 0.02, counts=None) -> Contiguous:
    """Per-expert token counts uniform in [count_lo, count_hi] (inclusive), each segment padded
    up to a multiple of 128 with rows whose expert index is -1.  Draw order: counts, A (all
    rows, padding included), B per expert."""
    g = _gen(seed)
    if counts is None:
        counts = torch.randint(count_lo, count_hi + 1, (G,), generator=g).numpy()
    counts = np.asarray(counts, dtype=np.int64)
    padded = (counts + BLOCK - 1) // BLOCK * BLOCK
    M_total = int(padded.sum())
    m_idx = np.full(M_total, -1, np.int32)
    off = 0
    for e in range(G):
        m_idx[off:off + counts[e]] = e
        off += int(padded[e])
    A = torch.randn(M_total, K, generator=g) * a_std
    a, sa = quantise_rows_1x128(A)
    b, sb = _grouped_b(G, N, K, b_std, g)
    return Contiguous(G, N, K, counts, m_idx, a, sa, b, sb)


def masked(G: int, M_max: int, N: int, K: int, seed: int, expected_m: int = 128,
           a_std: float = 1.0, b_std: float = 0.02, masked_m=None) -> Masked:
    """masked_m[g] uniform in [0, M_max] (inclusive); every row of A is filled, valid or not.
    Draw order: masked_m, A, B per expert."""
    g = _gen(seed)
    if masked_m is None:
        masked_m = torch.randint(0, M_max + 1, (G,), generator=g).numpy()
    masked_m = np.asarray(masked_m, dtype=np.int32)
    A = torch.randn(G * M_max, K, generator=g) * a_std
    a, sa = quantise_rows_1x128(A)
    a = a.reshape(G, M_max, K)
    sa = sa.reshape(G, M_max, K // BLOCK)
    b, sb = _grouped_b(G, N, K, b_std, g)
    return Masked(G, M_max, N, K, expected_m, masked_m, a, sa, b, sb)


def with_fp4_b(case, seed: int, b_std: float = 0.02):
    """A copy of a Dense / Contiguous / Masked case whose B is an FP4 (E2M1) operand: packed
    bytes [.., N, K/2] drawn uniformly (so every one of the 16 codes, -0 included, occurs in
    both nibble positions; element 2j of a row is the low nibble of byte j) and fresh 128x128
    block scales uniform in [0.5, 1.5] * b_std * 4/6 (the size an absmax/6 scaling of
    N(0, b_std^2) weights gives).  A, its scales and the layout fields are kept."""
    import dataclasses
    g = _gen(seed)
    b_shape = case.b.shape[:-1] + (case.b.shape[-1] // 2,)
    b = torch.randint(0, 256, b_shape, generator=g, dtype=torch.int32).to(torch.uint8).numpy()
    sb = ((torch.rand(case.sb.shape, generator=g) + 0.5) * (b_std * 4.0 / 6.0)).float().numpy()
    return dataclasses.replace(case, b=b, sb=sb)


# ---- edge-value inputs ---------------------------------------------------------------------
# Codes and scales drawn directly (no fp32 source, no quantisation) so that the inputs reach the
# values two-level accumulation exists for: products that cancel inside one 128-wide K slice,
# slices whose sums pass fp32's exact-integer range, every finite code including subnormals,
# and block scales whose products span 2^-60 .. 2^60.

E4M3_POS_MAX = 0x7E          # +448
E4M3_NAN = 0x7F              # the two NaN codes are 0x7F and 0xFF
E4M3_FINITE = np.array([c for c in range(256) if (c & 0x7F) != E4M3_NAN], np.uint8)  # 254 codes
E2M1_POS_MAX = 0x7           # +6 (sign in bit 3)
EDGE_PATTERNS = ("cancel", "cancel_residual", "pm_max", "all_codes")


def pack_e2m1(nibbles: np.ndarray) -> np.ndarray:
    """E2M1 codes [..., K] (one per uint8, low 4 bits) -> packed bytes [..., K/2], element 2j in
    the low nibble of byte j."""
    n = np.asarray(nibbles, np.uint8) & 0xF
    return (n[..., 0::2] | (n[..., 1::2] << 4)).astype(np.uint8)


def _signed(rng, mag_codes: np.ndarray, sign_bit: int) -> np.ndarray:
    signs = rng.integers(0, 2, mag_codes.shape).astype(np.uint8) * np.uint8(sign_bit)
    return (mag_codes.astype(np.uint8) | signs).astype(np.uint8)


def _edge_codes(pattern: str, rows: int, K: int, rng, fp4: bool, cancel_k, big_sign, second_sign):
    """Codes [rows, K] of one operand.  fp4: E2M1 codes (one per byte), else E4M3 codes.
    cancel_k[kb] = (k0, k1): the two positions of K block kb that carry the largest magnitude;
    big_sign [rows] (0/1) is the sign of the first, second_sign [rows] that of the second."""
    sign_bit = 0x8 if fp4 else 0x80
    big = E2M1_POS_MAX if fp4 else E4M3_POS_MAX
    if pattern == "all_codes":
        pool = np.arange(16, dtype=np.uint8) if fp4 else E4M3_FINITE
        return pool[rng.integers(0, pool.size, (rows, K))]
    if pattern == "pm_max":
        return _signed(rng, np.full((rows, K), big, np.uint8), sign_bit)
    # cancel / cancel_residual: small magnitudes everywhere (E4M3: subnormals 2^-9 .. 7 * 2^-9
    # and the smallest normals; E2M1: 0.5 .. 1.5), the largest magnitude at k0 and k1
    lo, hi = (1, 3) if fp4 else (1, 12)
    c = _signed(rng, rng.integers(lo, hi + 1, (rows, K)).astype(np.uint8), sign_bit)
    for kb, (k0, k1) in enumerate(cancel_k):
        c[:, k0] = big | (big_sign * sign_bit)
        c[:, k1] = big | (second_sign * sign_bit)
    return c.astype(np.uint8)


def edge_dense(pattern: str, M: int, N: int, K: int, seed: int, fp4: bool = False,
               scale_exp: int = 30) -> Dense:
    """A Dense case with edge-value codes (see EDGE_PATTERNS):
      cancel          per K block, positions k0 != k1 hold +-448 in A (the same sign at both)
                      and +-448 / -+448 in B (opposite signs), so the two largest products of
                      every slice cancel exactly; every other product is tiny (subnormal
                      codes), so the slice's sum is far below its magnitude;
      cancel_residual the same with B's second large code one step smaller (E4M3 416, E2M1
                      4): the slice keeps a residual (448 * 32, or 448 * 2) next to the tiny
                      products;
      pm_max          every code +-448 (E2M1: +-6): a slice of equal signs sums to 128 * 448^2,
                      past fp32's exact-integer range 2^24;
      all_codes       codes uniform over the 254 finite E4M3 codes (E2M1: all 16 codes).
    Scales are powers of two 2^U{-scale_exp .. scale_exp} per 1x128 A tile and per 128x128 B
    block, so sa * sb spans 2^-60 .. 2^60 at the default.  fp4: B is a packed E2M1 operand
    [N, K/2] (A stays E4M3).  Draw order: positions, signs, A, B, sa, sb."""
    assert pattern in EDGE_PATTERNS and K % BLOCK == 0
    rng = np.random.default_rng(seed)
    Kb, Nb = K // BLOCK, -(-N // BLOCK)
    cancel_k = []
    for kb in range(Kb):
        k0, k1 = rng.choice(BLOCK, 2, replace=False)
        cancel_k.append((kb * BLOCK + int(k0), kb * BLOCK + int(k1)))
    sa_sign = rng.integers(0, 2, (M,)).astype(np.uint8)
    sb_sign = rng.integers(0, 2, (N,)).astype(np.uint8)
    a = _edge_codes(pattern, M, K, rng, False, cancel_k, sa_sign, sa_sign)
    b = _edge_codes(pattern, N, K, rng, fp4, cancel_k, sb_sign, 1 - sb_sign)
    if pattern == "cancel_residual":
        smaller = 0x6 if fp4 else 0x7D       # E2M1 4 (the step below 6), E4M3 416
        for k0, k1 in cancel_k:
            b[:, k1] = (b[:, k1] & (0x8 if fp4 else 0x80)) | smaller
    sa = np.ldexp(1.0, rng.integers(-scale_exp, scale_exp + 1, (M, Kb))).astype(np.float32)
    sb = np.ldexp(1.0, rng.integers(-scale_exp, scale_exp + 1, (Nb, Kb))).astype(np.float32)
    if fp4:
        b = pack_e2m1(b)
    return Dense(M, N, K, a, sa, b, sb)


def edge_contiguous(pattern: str, N: int, K: int, seed: int, rows: int = 200, fp4: bool = False) -> Contiguous:
    """One expert segment (expert 1 of G = 2; expert 0 has no rows) of ``rows`` edge-value
    rows, padded to a multiple of 128 with -1 rows."""
    d = edge_dense(pattern, rows, N, K, seed, fp4=fp4)
    M_total = -(-rows // BLOCK) * BLOCK
    a = np.zeros((M_total, K), np.uint8)
    sa = np.ones((M_total, K // BLOCK), np.float32)
    a[:rows], sa[:rows] = d.a, d.sa
    mi = np.full(M_total, -1, np.int32)
    mi[:rows] = 1
    b = np.stack([np.zeros_like(d.b), d.b])
    sb = np.stack([np.ones_like(d.sb), d.sb])
    return Contiguous(2, N, K, np.array([0, rows], np.int64), mi, a, sa, b, sb)


def edge_masked(pattern: str, N: int, K: int, seed: int, rows: int = 200, M_max: int = 256,
                fp4: bool = False) -> Masked:
    """One masked group (group 1 of G = 2 holds ``rows`` valid edge-value rows; group 0 has
    none); rows past masked_m are filled too."""
    d = edge_dense(pattern, M_max, N, K, seed, fp4=fp4)
    a = np.stack([np.zeros_like(d.a), d.a])
    sa = np.stack([np.ones_like(d.sa), d.sa])
    b = np.stack([np.zeros_like(d.b), d.b])
    sb = np.stack([np.ones_like(d.sb), d.sb])
    return Masked(2, M_max, N, K, rows, np.array([0, rows], np.int32), a, sa, b, sb)


# ---- the named workloads ----------------------------------------------------------------

SMALL_DENSE = dict(M=128, N=256, K=512)
SWEEP_NK = [(2112, 7168), (24576, 1536), (7168, 16384), (4096, 7168), (7168, 2048)]
SWEEP_M = [64, 128, 4096]
CONTIG = dict(G=8, N=4096, K=7168)
MASKED = dict(G=32, M_max=256, N=4096, K=7168, expected_m=128)
PREFILL = dict(M=8192, N=7168, K=18432)


def small_dense(seed: int = 1000) -> Dense:
    """128x256x512, A and B ~ N(0,1)."""
    return dense(**SMALL_DENSE, seed=seed)


def sweep_shapes():
    """The fifteen (M, N, K) shapes of the dense sweep, M-major."""
    return [(m, n, k) for m in SWEEP_M for (n, k) in SWEEP_NK]


def sweep_case(i: int) -> Dense:
    """Shape i of the dense sweep: A ~ N(0,1), B ~ N(0, 0.02^2)."""
    M, N, K = sweep_shapes()[i]
    return dense(M, N, K, seed=2000 + i, a_std=1.0, b_std=0.02)


def contiguous_case(seed: int = 3000) -> Contiguous:
    return contiguous(**CONTIG, seed=seed)


def masked_case(seed: int = 4000) -> Masked:
    return masked(**MASKED, seed=seed)


def prefill_case(seed: int = 5000) -> Dense:
    """8192x7168x18432 with ~1% outliers x50 in A."""
    return dense(**PREFILL, seed=seed, a_std=1.0, b_std=0.02, outlier_frac=0.01)
