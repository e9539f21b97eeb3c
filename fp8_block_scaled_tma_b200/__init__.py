"""Python binding of the B200 (sm_100a) FP8 block-scaled NT GEMM library.

Argument marshalling only: each function checks shapes and dtypes of torch tensors and calls
the C ABI of ``libdg_b200.so`` (declared in ``include/dg.h``) with their device pointers and
the current CUDA stream.  Every step of the computation runs in the library's CUDA kernels;
there is no fallback.  Importing this package fails loudly when the library is not built.

Entry points (the names of the DeepGEMM release write-up, "如何使用"):
  dg_gemm_fp8_fp8_bf16_nt                        dense NT GEMM
  dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous   MoE grouped GEMM, contiguous layout
  dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked       MoE grouped GEMM, masked layout
plus the SM-count and TMA-alignment utilities.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg_b200.so")

DG_OK = 0
DG_ERR_INVALID_ARG = -1
DG_ERR_UNSUPPORTED = -2
DG_ERR_CUDA = -3
DG_ERR_TIMEOUT = -4
DG_ERR_WORKSPACE = -5
DG_ERR_LAYOUT = -6

BLOCK = 128


class DGError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build the CUDA library first "
            "(python fp8_block_scaled_tma_b200/build.py, or __graft_entry__.build())")
    lib = ctypes.CDLL(LIB_PATH)
    vp, fp, ip, i, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.dg_gemm_fp8_fp8_bf16_nt.argtypes = [vp, fp, vp, fp, vp, i, i, i, vp, sz, vp]
    lib.dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous.argtypes = [vp, fp, vp, fp, vp, ip, i, i, i,
                                                                 i, vp, sz, vp]
    lib.dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked.argtypes = [vp, fp, vp, fp, vp, ip, i, i, i, i,
                                                             i, vp, sz, vp]
    lib.dg_gemm_fp8_fp4_bf16_nt.argtypes = [vp, fp, vp, fp, vp, i, i, i, vp]
    lib.dg_gemm_fp8_fp8_bf16_nt_noalloc.argtypes = [vp, fp, vp, fp, vp, i, i, i, vp]
    lib.dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous.argtypes = [vp, fp, vp, fp, vp, ip, i, i, i,
                                                                 i, vp]
    lib.dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked.argtypes = [vp, fp, vp, fp, vp, ip, i, i, i, i,
                                                             i, vp]
    for name in ("dg_gemm_fp8_fp8_bf16_nt", "dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous",
                 "dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked", "dg_gemm_fp8_fp4_bf16_nt",
                 "dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous",
                 "dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked", "dg_gemm_fp8_fp8_bf16_nt_noalloc"):
        getattr(lib, name).restype = ctypes.c_int
    lib.dg_set_num_sms.argtypes = [i]
    lib.dg_set_num_sms.restype = i
    lib.dg_get_num_sms.argtypes = []
    lib.dg_get_num_sms.restype = i
    lib.dg_get_tma_aligned_size.argtypes = [i, i]
    lib.dg_get_tma_aligned_size.restype = i
    lib.dg_get_workspace_size.argtypes = [i, i, i, i, i]
    lib.dg_get_workspace_size.restype = sz
    lib.dg_status_string.argtypes = [i]
    lib.dg_status_string.restype = ctypes.c_char_p
    lib.dg_poll_device_error.argtypes = [vp]
    lib.dg_poll_device_error.restype = i
    lib.dg_set_wait_timeout_ns.argtypes = [ctypes.c_ulonglong]
    lib.dg_set_wait_timeout_ns.restype = ctypes.c_ulonglong
    lib.dg_set_config_override.argtypes = [i, i, i]
    lib.dg_set_config_override.restype = i
    lib.dg_set_fault_injection.argtypes = [i]
    lib.dg_set_fault_injection.restype = i
    lib.dg_set_kernel_family.argtypes = [i]
    lib.dg_set_kernel_family.restype = i
    lib.dg_quantize_fp8_1x128.argtypes = [vp, vp, fp, i, i, vp]
    lib.dg_swiglu_quantize_fp8_1x128.argtypes = [vp, vp, fp, i, i, ip, i, vp]
    lib.dg_swiglu_quantize_fp8_1x128.restype = i
    lib.dg_quantize_fp8_1x128.restype = i
    lib.dg_set_tensor_map_cache.argtypes = [i]
    lib.dg_set_tensor_map_cache.restype = i
    lib.dg_get_tensor_map_cache_stats.argtypes = [ctypes.POINTER(ctypes.c_ulonglong),
                                                  ctypes.POINTER(ctypes.c_ulonglong)]
    lib.dg_get_tensor_map_cache_stats.restype = i
    lib.dg_set_pdl.argtypes = [i]
    lib.dg_set_pdl.restype = i
    ipp = ctypes.POINTER(ctypes.c_int)
    lib.dg_get_last_launch.argtypes = [ipp, ipp, ipp, ipp, ipp, ipp]
    lib.dg_get_last_launch.restype = i
    return lib


lib = _load()


# ---- helpers ------------------------------------------------------------------------------

def status_string(status: int) -> str:
    return lib.dg_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != DG_OK:
        raise DGError(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _fp8(t: torch.Tensor, name: str) -> None:
    if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise TypeError(f"{name} must hold e4m3 codes (uint8 or float8_e4m3fn), got {t.dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def _fp4(t: torch.Tensor, name: str) -> None:
    fp4_x2 = getattr(torch, "float4_e2m1fn_x2", None)
    if t.dtype != torch.uint8 and t.dtype != fp4_x2:
        raise TypeError(f"{name} must hold packed e2m1 pairs (uint8 or float4_e2m1fn_x2), got {t.dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if t.data_ptr() % 32 != 0:
        raise ValueError(f"{name} must be 32-byte aligned")


def _f32(t: torch.Tensor, name: str, shape) -> None:
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _out(t: torch.Tensor, shape) -> None:
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError("d must be a contiguous bfloat16 CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"d has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _i32(t: torch.Tensor, name: str, shape) -> None:
    if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def get_tma_aligned_size(x: int, elem_bytes: int) -> int:
    r = lib.dg_get_tma_aligned_size(int(x), int(elem_bytes))
    if r < 0:
        raise DGError(r, "dg_get_tma_aligned_size")
    return r


def set_num_sms(n: int) -> int:
    return lib.dg_set_num_sms(int(n))


def get_num_sms() -> int:
    r = lib.dg_get_num_sms()
    if r < 0:
        raise DGError(r, "dg_get_num_sms")
    return r


def get_workspace_size(kind: int, M: int, N: int, K: int, G: int = 1) -> int:
    """Bytes of workspace the stream-K kernel (kernel family 5, dense M <= 64) needs for this
    call (0: it does not apply).  Allocate it zero-filled, e.g. with workspace_for, and keep one
    per stream.  Automatic mode never needs one."""
    return int(lib.dg_get_workspace_size(kind, M, N, K, G))


def workspace_for(M: int, N: int, K: int, device=None):
    """A zero-filled workspace for dense calls of this size on the current device (None when
    the call uses none)."""
    n = get_workspace_size(0, M, N, K)
    if n == 0:
        return None
    return torch.zeros(n, dtype=torch.uint8, device=device if device is not None else "cuda")


def poll_device_error(stream=None) -> int:
    return lib.dg_poll_device_error(_stream(stream))


def set_wait_timeout_ns(ns: int) -> int:
    return int(lib.dg_set_wait_timeout_ns(int(ns)))


def set_config_override(block_n: int = 0, num_stages: int = 0, splits: int = 0) -> None:
    _check(lib.dg_set_config_override(int(block_n), int(num_stages), int(splits)),
           "dg_set_config_override")


def set_fault_injection(mode: int) -> int:
    """Test hook: 1 makes the MMA issuer wait on a barrier nothing signals (the watchdog then
    reports DG_ERR_TIMEOUT); 0 turns it off.  Returns the previous mode."""
    r = lib.dg_set_fault_injection(int(mode))
    if r < 0:
        raise DGError(r, "dg_set_fault_injection")
    return r


FAMILY_AUTO, FAMILY_ONE_CTA, FAMILY_PAIR, FAMILY_SPLIT_K = 0, 1, 2, 3


def set_kernel_family(family: int) -> int:
    """0 automatic, 1 one-CTA kernels, 2 CTA-pair kernels where the layout allows, 3 split-K
    cluster kernel for dense calls, 4 swapped-operand kernel for dense calls with M <= 128,
    5 stream-K swapped-operand kernel for dense calls with M <= 64 (needs the workspace of
    get_workspace_size).  Returns the previous value."""
    r = lib.dg_set_kernel_family(int(family))
    if r < 0:
        raise DGError(r, "dg_set_kernel_family")
    return r


def set_pdl(enable: bool) -> bool:
    """Programmatic dependent launch of the GEMMs (on by default): back-to-back kernels overlap
    their on-chip set-up with the previous kernel's tail.  Returns the previous setting."""
    r = lib.dg_set_pdl(1 if enable else 0)
    if r < 0:
        raise DGError(r, "dg_set_pdl")
    return bool(r)


def set_tensor_map_cache(enable: bool) -> bool:
    """Turns the cache of encoded TMA tensor maps on or off (off drops every entry).  Returns
    the previous setting."""
    r = lib.dg_set_tensor_map_cache(1 if enable else 0)
    if r < 0:
        raise DGError(r, "dg_set_tensor_map_cache")
    return bool(r)


def tensor_map_cache_stats() -> tuple[int, int]:
    """(hits, misses) of the tensor-map cache since the library was loaded."""
    h, m = ctypes.c_ulonglong(), ctypes.c_ulonglong()
    _check(lib.dg_get_tensor_map_cache_stats(ctypes.byref(h), ctypes.byref(m)),
           "dg_get_tensor_map_cache_stats")
    return h.value, m.value


def get_last_launch() -> dict:
    v = [ctypes.c_int() for _ in range(6)]
    _check(lib.dg_get_last_launch(*[ctypes.byref(x) for x in v]), "dg_get_last_launch")
    return dict(block_n=v[0].value, stages=v[1].value, grid=v[2].value, tiles=v[3].value,
                family=v[4].value, splits=v[5].value)


def sfa_mn_major(sa: torch.Tensor) -> torch.Tensor:
    """Layout marshalling of A's scales: logical [rows, K/128] (or [G, rows, K/128]) fp32 ->
    the MN-major, TMA-aligned layout the kernels read: [K/128, align4(rows)] (or
    [G, K/128, align4(rows)]), zero in the padding."""
    sa = sa.float()
    if sa.dim() == 2:
        rows, kb = sa.shape
        out = torch.zeros(kb, get_tma_aligned_size(rows, 4), dtype=torch.float32, device=sa.device)
        out[:, :rows] = sa.t()
        return out
    if sa.dim() == 3:
        g, rows, kb = sa.shape
        out = torch.zeros(g, kb, get_tma_aligned_size(rows, 4), dtype=torch.float32,
                          device=sa.device)
        out[:, :, :rows] = sa.transpose(1, 2)
        return out
    raise ValueError("sa must be 2-D or 3-D")


# ---- the three GEMMs ------------------------------------------------------------------------

def dg_gemm_fp8_fp8_bf16_nt(a, sfa, b, sfb, d, workspace=None, stream=None) -> None:
    """d[M,N] (bf16) = a[M,K] (e4m3) . b[N,K]^T with sfa [K/128, align4(M)] (MN-major) and
    sfb [ceil(N/128), K/128]."""
    _fp8(a, "a")
    _fp8(b, "b")
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b disagree on K")
    _f32(sfa, "sfa", (K // BLOCK, get_tma_aligned_size(M, 4)))
    _f32(sfb, "sfb", (-(-N // BLOCK), K // BLOCK))
    _out(d, (M, N))
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.dg_gemm_fp8_fp8_bf16_nt(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), M, N, K,
                                       _ptr(workspace), ws, _stream(stream)),
           "dg_gemm_fp8_fp8_bf16_nt")


def dg_gemm_fp8_fp8_bf16_nt_noalloc(a, sfa, b, sfb, d, stream=None) -> None:
    """dg_gemm_fp8_fp8_bf16_nt for callers that cannot allocate device memory: the stream-K
    kernel with its scratch in an array built into the library (dense, M <= 64; see dg.h)."""
    _fp8(a, "a")
    _fp8(b, "b")
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b disagree on K")
    _f32(sfa, "sfa", (K // BLOCK, get_tma_aligned_size(M, 4)))
    _f32(sfb, "sfb", (-(-N // BLOCK), K // BLOCK))
    _out(d, (M, N))
    _check(lib.dg_gemm_fp8_fp8_bf16_nt_noalloc(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), M, N, K,
                                               _stream(stream)),
           "dg_gemm_fp8_fp8_bf16_nt_noalloc")


def quantize_fp8_1x128(x, q=None, sfa=None, stream=None):
    """Per-token FP8 quantisation on the GPU: x bf16 [M,K] -> (q uint8 e4m3 codes [M,K],
    sfa fp32 [K/128, align4(M)] MN-major, the GEMMs' A-scale layout).  Output tensors may be
    passed in (they are overwritten); otherwise they are allocated here with torch."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous() or x.dim() != 2:
        raise ValueError("x must be a contiguous 2-D bfloat16 CUDA tensor")
    M, K = x.shape
    if K % BLOCK != 0:
        raise ValueError("K must be a multiple of 128")
    if q is None:
        q = torch.empty(M, K, dtype=torch.uint8, device=x.device)
    _fp8(q, "q")
    if tuple(q.shape) != (M, K):
        raise ValueError("q must be [M, K]")
    if sfa is None:
        sfa = torch.empty(K // BLOCK, get_tma_aligned_size(M, 4), dtype=torch.float32, device=x.device)
    _f32(sfa, "sfa", (K // BLOCK, get_tma_aligned_size(M, 4)))
    _check(lib.dg_quantize_fp8_1x128(_ptr(x), _ptr(q), _ptr(sfa), M, K, _stream(stream)),
           "dg_quantize_fp8_1x128")
    return q, sfa


def swiglu_quantize_fp8_1x128(h, masked_m=None, rows_per_group=0, q=None, sfa=None, stream=None):
    """SwiGLU (gate half, then up half of each row of h bf16 [M, 2I]) followed by the per-token
    FP8 quantisation.  Returns (q uint8 [M, I], sfa fp32): [I/128, align4(M)] without masked_m,
    [G, I/128, align4(rows_per_group)] with it (the masked GEMM's layout)."""
    if h.dtype != torch.bfloat16 or not h.is_cuda or not h.is_contiguous() or h.dim() != 2:
        raise ValueError("h must be a contiguous 2-D bfloat16 CUDA tensor")
    M, two_i = h.shape
    I = two_i // 2
    if two_i % 2 or I % BLOCK:
        raise ValueError("h must be [M, 2I] with I a multiple of 128")
    if q is None:
        q = torch.empty(M, I, dtype=torch.uint8, device=h.device)
    _fp8(q, "q")
    if masked_m is not None:
        if rows_per_group <= 0 or M % rows_per_group:
            raise ValueError("rows_per_group must divide M")
        G = M // rows_per_group
        if masked_m.dtype != torch.int32 or tuple(masked_m.shape) != (G,) or not masked_m.is_cuda:
            raise ValueError("masked_m must be an int32 CUDA tensor of G entries")
        shape = (G, I // BLOCK, get_tma_aligned_size(rows_per_group, 4))
    else:
        shape = (I // BLOCK, get_tma_aligned_size(M, 4))
    if sfa is None:
        sfa = torch.empty(shape, dtype=torch.float32, device=h.device)
    _f32(sfa, "sfa", shape)
    _check(lib.dg_swiglu_quantize_fp8_1x128(_ptr(h), _ptr(q), _ptr(sfa), M, I, _ptr(masked_m),
                                            int(rows_per_group), _stream(stream)),
           "dg_swiglu_quantize_fp8_1x128")
    return q, sfa


def dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(a, sfa, b, sfb, d, m_indices, workspace=None,
                                                 stream=None) -> None:
    """Contiguous-layout grouped GEMM: a [M_total,K], sfa [K/128, M_total], b [G,N,K],
    sfb [G, ceil(N/128), K/128], d [M_total,N], m_indices int32 [M_total] (-1 = padding)."""
    _fp8(a, "a")
    _fp8(b, "b")
    M, K = a.shape
    G, N, Kb_ = b.shape
    if Kb_ != K:
        raise ValueError("a and b disagree on K")
    _f32(sfa, "sfa", (K // BLOCK, get_tma_aligned_size(M, 4)))
    _f32(sfb, "sfb", (G, -(-N // BLOCK), K // BLOCK))
    _out(d, (M, N))
    _i32(m_indices, "m_indices", (M,))
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(
        _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), _ptr(m_indices), M, N, K, G,
        _ptr(workspace), ws, _stream(stream)), "dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous")


def dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(a, sfa, b, sfb, d, masked_m, expected_m: int,
                                             workspace=None, stream=None) -> None:
    """Masked-layout grouped GEMM: a [G,M_max,K], sfa [G, K/128, align4(M_max)], b [G,N,K],
    sfb [G, ceil(N/128), K/128], d [G,M_max,N], masked_m int32 [G]."""
    _fp8(a, "a")
    _fp8(b, "b")
    G, M_max, K = a.shape
    Gb, N, Kb_ = b.shape
    if Gb != G or Kb_ != K:
        raise ValueError("a and b disagree on G or K")
    _f32(sfa, "sfa", (G, K // BLOCK, get_tma_aligned_size(M_max, 4)))
    _f32(sfb, "sfb", (G, -(-N // BLOCK), K // BLOCK))
    _out(d, (G, M_max, N))
    _i32(masked_m, "masked_m", (G,))
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(
        _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), _ptr(masked_m), G, M_max, N, K,
        int(expected_m), _ptr(workspace), ws, _stream(stream)),
        "dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked")


# ---- FP8 x FP4: b holds packed E2M1 pairs, [.., N, K/2] bytes, element 2j in the low nibble --

def dg_gemm_fp8_fp4_bf16_nt(a, sfa, b, sfb, d, stream=None) -> None:
    """d[M,N] (bf16) = a[M,K] (e4m3) . b^T, b packed e2m1 [N, K/2] bytes; scales as in
    dg_gemm_fp8_fp8_bf16_nt."""
    _fp8(a, "a")
    _fp4(b, "b")
    M, K = a.shape
    N = b.shape[0]
    if 2 * b.shape[1] != K:
        raise ValueError("b must be [N, K/2] packed bytes")
    _f32(sfa, "sfa", (K // BLOCK, get_tma_aligned_size(M, 4)))
    _f32(sfb, "sfb", (-(-N // BLOCK), K // BLOCK))
    _out(d, (M, N))
    _check(lib.dg_gemm_fp8_fp4_bf16_nt(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), M, N, K,
                                       _stream(stream)), "dg_gemm_fp8_fp4_bf16_nt")


def dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous(a, sfa, b, sfb, d, m_indices, stream=None) -> None:
    """Contiguous-layout grouped FP8 x FP4 GEMM: b packed e2m1 [G, N, K/2] bytes; everything
    else as in dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous."""
    _fp8(a, "a")
    _fp4(b, "b")
    M, K = a.shape
    G, N, half_k = b.shape
    if 2 * half_k != K:
        raise ValueError("b must be [G, N, K/2] packed bytes")
    _f32(sfa, "sfa", (K // BLOCK, get_tma_aligned_size(M, 4)))
    _f32(sfb, "sfb", (G, -(-N // BLOCK), K // BLOCK))
    _out(d, (M, N))
    _i32(m_indices, "m_indices", (M,))
    _check(lib.dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous(
        _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), _ptr(m_indices), M, N, K, G,
        _stream(stream)), "dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous")


def dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked(a, sfa, b, sfb, d, masked_m, expected_m: int,
                                             stream=None) -> None:
    """Masked-layout grouped FP8 x FP4 GEMM: b packed e2m1 [G, N, K/2] bytes; everything else
    as in dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked."""
    _fp8(a, "a")
    _fp4(b, "b")
    G, M_max, K = a.shape
    Gb, N, half_k = b.shape
    if Gb != G or 2 * half_k != K:
        raise ValueError("b must be [G, N, K/2] packed bytes with a's G")
    _f32(sfa, "sfa", (G, K // BLOCK, get_tma_aligned_size(M_max, 4)))
    _f32(sfb, "sfb", (G, -(-N // BLOCK), K // BLOCK))
    _out(d, (G, M_max, N))
    _i32(masked_m, "masked_m", (G,))
    _check(lib.dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked(
        _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), _ptr(masked_m), G, M_max, N, K,
        int(expected_m), _stream(stream)), "dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked")
