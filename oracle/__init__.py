"""CPU oracle for the FP8 block-scaled NT GEMM (dense, contiguous-grouped, masked-grouped).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  The product path (the CUDA library and its
Python binding) never imports, links or runs it, and this package imports nothing from the
product.  The arithmetic lives in ``oracle.c`` (plain C, fp64); this module only loads the
shared object and marshals numpy arrays.

What the oracle computes follows the DeepGEMM release write-up ("深入了解DeepGEMM": FP8 GEMM
with DeepSeek-V3 fine-grained scaling; "如何使用": the NT layout and the two grouped MoE
layouts).  Every function here has a pin in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

BLOCK = 128

_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` with gcc (no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
               "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    u8p = ctypes.POINTER(ctypes.c_uint8)
    f32p = ctypes.POINTER(ctypes.c_float)
    i32p = ctypes.POINTER(ctypes.c_int32)
    i64p = ctypes.POINTER(ctypes.c_int64)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    f64p = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
    lib.orc_e4m3_encode.restype = ctypes.c_uint8
    lib.orc_quantize_1x128.argtypes = [ctypes.POINTER(ctypes.c_uint16), ctypes.c_int64, ctypes.c_int64,
                                       ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_float)]
    lib.orc_quantize_1x128.restype = ctypes.c_int
    lib.orc_swiglu_quantize.argtypes = [ctypes.POINTER(ctypes.c_uint16), ctypes.c_int64, ctypes.c_int64,
                                        ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_uint8),
                                        ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]
    lib.orc_swiglu_quantize.restype = ctypes.c_int
    lib.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
    lib.orc_e2m1_decode.restype = ctypes.c_double
    lib.orc_e2m1_to_e4m3.argtypes = [ctypes.POINTER(ctypes.c_uint8), ctypes.c_int64, ctypes.c_int64,
                                     ctypes.POINTER(ctypes.c_uint8)]
    lib.orc_e2m1_to_e4m3.restype = None
    lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3_decode.restype = ctypes.c_double
    lib.orc_bf16_rne.argtypes = [ctypes.c_double]
    lib.orc_bf16_rne.restype = ctypes.c_uint16
    lib.orc_gemm_dense_rows.argtypes = [u8p, f32p, u8p, f32p, i64, i64, i64, i64p, i64, u16p,
                                        f64p, f64p, ctypes.c_int]
    lib.orc_gemm_dense_rows.restype = ctypes.c_int
    lib.orc_gemm_contiguous.argtypes = [u8p, f32p, u8p, f32p, i32p, i64, i64, i64, i64, i64p,
                                        i64, u16p, f64p, f64p, ctypes.c_int]
    lib.orc_gemm_contiguous.restype = ctypes.c_int
    lib.orc_gemm_masked.argtypes = [u8p, f32p, u8p, f32p, i32p, i64, i64, i64, i64, i64p, i64,
                                    u16p, f64p, f64p, ctypes.c_int]
    lib.orc_gemm_masked.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(arr: np.ndarray | None, ctype):
    if arr is None:
        return ctypes.cast(None, ctypes.POINTER(ctype))
    assert arr.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return arr.ctypes.data_as(ctypes.POINTER(ctype))


def _as(x, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x), dtype=dtype)


def e4m3_decode(code: int) -> float:
    """Value of one OCP E4M3 ("fn") code, from the format's definition."""
    return float(_load().orc_e4m3_decode(int(code) & 0xFF))


def e4m3_encode(x: float) -> int:
    """fp32 -> E4M3 code, round to nearest even, saturating at 448."""
    return int(_load().orc_e4m3_encode(float(x)))


def quantize_1x128(x_bits: np.ndarray):
    """Per-token FP8 quantisation.  x_bits: uint16 bf16 bits [M][K].  Returns (codes uint8
    [M][K], scales float32 [M][K/128])."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    sa = np.empty((M, K // 128), dtype=np.float32)
    r = _load().orc_quantize_1x128(x.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)), M, K,
                                   q.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                   sa.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    if r != 0:
        raise ValueError("orc_quantize_1x128: K must be a multiple of 128")
    return q, sa


def swiglu_quantize(h_bits: np.ndarray, row_valid: np.ndarray | None = None):
    """SwiGLU then per-token FP8 quantisation.  h_bits: uint16 bf16 bits [M][2I] (gate half,
    then up half).  Returns (codes uint8 [M][I], scales float32 [M][I/128], y float32 [M][I]);
    rows with row_valid == 0 are left as 0 / 0 / NaN."""
    h = np.ascontiguousarray(h_bits, dtype=np.uint16)
    M, two_i = h.shape
    I = two_i // 2
    q = np.zeros((M, I), dtype=np.uint8)
    sa = np.zeros((M, I // 128), dtype=np.float32)
    y = np.full((M, I), np.nan, dtype=np.float32)
    rv = None
    if row_valid is not None:
        rv = np.ascontiguousarray(row_valid, dtype=np.uint8)
    r = _load().orc_swiglu_quantize(h.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)), M, I,
                                    None if rv is None else rv.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                    q.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                    sa.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                    y.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    if r != 0:
        raise ValueError("orc_swiglu_quantize: I must be a multiple of 128")
    return q, sa, y


def e2m1_decode(nibble: int) -> float:
    return float(_load().orc_e2m1_decode(int(nibble) & 0xF))


def e2m1_to_e4m3(packed: np.ndarray) -> np.ndarray:
    """Packed E2M1 [..., rows, K/2] (element 2j in the low nibble of byte j) -> E4M3 codes
    [..., rows, K] of the same values."""
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    lead, half_k = p.shape[:-1], p.shape[-1]
    rows = int(np.prod(lead)) if lead else 1
    out = np.empty(lead + (2 * half_k,), dtype=np.uint8)
    _load().orc_e2m1_to_e4m3(p.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), rows, 2 * half_k,
                             out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    return out


def bf16_rne(x: float) -> int:
    """Bit pattern of ``x`` rounded once to bfloat16, nearest-even."""
    return int(_load().orc_bf16_rne(float(x)))


class Result:
    """Oracle output: ``bits`` (uint16 bf16 patterns), ``acc`` (fp64 value before rounding),
    ``mag`` (fp64 sum of |sa a| |sb b| per element, used by the tolerance)."""

    def __init__(self, bits, acc, mag):
        self.bits, self.acc, self.mag = bits, acc, mag

    @property
    def value(self) -> np.ndarray:
        """The bf16 results widened to float64."""
        return bf16_bits_to_f64(self.bits)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns exactly (bf16 is the top half of an fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def gemm_dense(a, sa, b, sb, rows=None, threads: int = 0) -> Result:
    """D = A . B^T for A [M,K] e4m3 codes (uint8) with scales sa [M,K/128] and B [N,K] codes
    with scales sb [ceil(N/128),K/128].  With ``rows`` only those rows of A are computed and
    the result has ``len(rows)`` rows in that order."""
    a = _as(a, np.uint8)
    b = _as(b, np.uint8)
    sa = _as(sa, np.float32)
    sb = _as(sb, np.float32)
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K or sa.shape != (M, K // BLOCK) or sb.shape != (-(-N // BLOCK), K // BLOCK):
        raise ValueError("shape mismatch")
    r = np.arange(M, dtype=np.int64) if rows is None else _as(rows, np.int64)
    bits = np.zeros((len(r), N), np.uint16)
    acc = np.zeros((len(r), N), np.float64)
    mag = np.zeros((len(r), N), np.float64)
    rc = _load().orc_gemm_dense_rows(_ptr(a, ctypes.c_uint8), _ptr(sa, ctypes.c_float),
                                     _ptr(b, ctypes.c_uint8), _ptr(sb, ctypes.c_float), M, N, K,
                                     _ptr(r, ctypes.c_int64), len(r), _ptr(bits, ctypes.c_uint16),
                                     _ptr(acc, ctypes.c_double), _ptr(mag, ctypes.c_double),
                                     threads)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return Result(bits, acc, mag)


def gemm_contiguous(a, sa, b, sb, m_indices, out_fill: int = 0xFFFF, rows=None,
                    threads: int = 0) -> Result:
    """Contiguous grouped GEMM: a [M_total,K], sa [M_total,K/128], b [G,N,K],
    sb [G,ceil(N/128),K/128], m_indices [M_total] int32 (expert, or -1 for padding).
    Output arrays are [M_total,N]; rows with -1 keep ``out_fill`` (bits) and NaN (acc, mag).
    ``rows`` limits the computation to a subset of rows (the others also keep the fill)."""
    a = _as(a, np.uint8)
    b = _as(b, np.uint8)
    sa = _as(sa, np.float32)
    sb = _as(sb, np.float32)
    mi = _as(m_indices, np.int32)
    M, K = a.shape
    G, N, _ = b.shape
    bits = np.full((M, N), out_fill, np.uint16)
    acc = np.full((M, N), np.nan, np.float64)
    mag = np.full((M, N), np.nan, np.float64)
    r = None if rows is None else _as(rows, np.int64)
    rc = _load().orc_gemm_contiguous(_ptr(a, ctypes.c_uint8), _ptr(sa, ctypes.c_float),
                                     _ptr(b, ctypes.c_uint8), _ptr(sb, ctypes.c_float),
                                     _ptr(mi, ctypes.c_int32), M, N, K, G,
                                     _ptr(r, ctypes.c_int64), 0 if r is None else len(r),
                                     _ptr(bits, ctypes.c_uint16), _ptr(acc, ctypes.c_double),
                                     _ptr(mag, ctypes.c_double), threads)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return Result(bits, acc, mag)


def gemm_masked(a, sa, b, sb, masked_m, out_fill: int = 0xFFFF, rows=None,
                threads: int = 0) -> Result:
    """Masked grouped GEMM: a [G,M_max,K], sa [G,M_max,K/128], b [G,N,K],
    sb [G,ceil(N/128),K/128], masked_m [G] int32.  Output arrays are [G,M_max,N]; rows
    r >= masked_m[g] keep ``out_fill`` / NaN.  ``rows`` are flattened g*M_max + r indices."""
    a = _as(a, np.uint8)
    b = _as(b, np.uint8)
    sa = _as(sa, np.float32)
    sb = _as(sb, np.float32)
    mm = _as(masked_m, np.int32)
    G, M_max, K = a.shape
    N = b.shape[1]
    bits = np.full((G, M_max, N), out_fill, np.uint16)
    acc = np.full((G, M_max, N), np.nan, np.float64)
    mag = np.full((G, M_max, N), np.nan, np.float64)
    r = None if rows is None else _as(rows, np.int64)
    rc = _load().orc_gemm_masked(_ptr(a, ctypes.c_uint8), _ptr(sa, ctypes.c_float),
                                 _ptr(b, ctypes.c_uint8), _ptr(sb, ctypes.c_float),
                                 _ptr(mm, ctypes.c_int32), G, M_max, N, K,
                                 _ptr(r, ctypes.c_int64), 0 if r is None else len(r),
                                 _ptr(bits, ctypes.c_uint16), _ptr(acc, ctypes.c_double),
                                 _ptr(mag, ctypes.c_double), threads)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return Result(bits, acc, mag)
