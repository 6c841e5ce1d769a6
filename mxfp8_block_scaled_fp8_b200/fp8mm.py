"""Python binding of ``libfp8mm.so`` (the C ABI in ``include/fp8mm.h``).

Argument marshalling only: every step of the quantizers and GEMMs runs in the
library's CUDA kernels.  torch supplies device memory and the current stream.
There is no fallback: if the library is missing or a call fails, an
``Fp8mmError`` is raised.

E4M3 operands are uint8 tensors holding the codes (a ``torch.float8_e4m3fn``
tensor is accepted too and viewed as uint8).  B is passed as [n, k] (K
contiguous), i.e. the transpose of the pages' logical [k, n].
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8mm.so")

FP8MM_OK = 0
FP8MM_ERR_DEVICE = 7
KERNEL_AUTO, KERNEL_TILED, KERNEL_SMALL_M, KERNEL_TILED_1SM, KERNEL_TILED_2SM, KERNEL_TILED_1SM_N128 = 0, 1, 2, 3, 4, 5


class Fp8mmError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        msg = f"{fn} failed: status {status}"
        if _lib is not None:
            msg += f" ({_lib.fp8mm_status_str(status).decode()})"
        if detail:
            msg += f"; {detail}"
        super().__init__(msg)


FLAG_WEIGHTS_READY = 1
FLAG_SPLIT_VIA_WORKSPACE = 2
FLAG_SF_A_8X4 = 4


class Opts(ctypes.Structure):
    _fields_ = [("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("kernel", ctypes.c_int32), ("small_m_ctas", ctypes.c_int32), ("flags", ctypes.c_uint32)]


_lib = None
_P, _I64, _U8P = ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p

_SIGNATURES = {
    "fp8_quantize_rowwise": ([_P, _I64, _I64, _I64, _P, _I64, _P, _P], ctypes.c_int),
    "mxfp8_quantize": ([_P, _I64, _I64, _I64, _P, _I64, _P, _P], ctypes.c_int),
    "fp8_gemm": ([_P, _P, _I64, _I64, _I64, _P, _P, _P, _I64, ctypes.POINTER(Opts), _P], ctypes.c_int),
    "fp8_tensor_scale": ([_P, _I64, _I64, _I64, _P, _P], ctypes.c_int),
    "fp8_quantize_static": ([_P, _I64, _I64, _I64, _P, _P, _I64, _P], ctypes.c_int),
    "fp8_gemm_e4m3_out": ([_P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _I64, ctypes.POINTER(Opts), _P], ctypes.c_int),
    "mxfp8_gemm": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _I64, ctypes.POINTER(Opts), _P], ctypes.c_int),
    "mxfp8_quantize_gemm": ([_P, _I64, _P, _P, _I64, _I64, _I64, _P, _I64, ctypes.POINTER(Opts), _P], ctypes.c_int),
    "concat_mla_k": ([_P, _P, _P] + [_I64] * 11 + [_P], ctypes.c_int),
    "fp8mm_sf_bytes": ([_I64, _I64], ctypes.c_size_t),
    "fp8mm_sf_offset": ([_I64, _I64, _I64, _I64], ctypes.c_int64),
    "fp8mm_sf8x4_bytes": ([_I64, _I64], ctypes.c_size_t),
    "fp8mm_sf8x4_offset": ([_I64, _I64, _I64, _I64], ctypes.c_int64),
    "mxfp8_quantize_8x4": ([_P, _I64, _I64, _I64, _P, _I64, _P, _P], ctypes.c_int),
    "fp8mm_sf_to_canonical": ([_P, _I64, _I64, _P], ctypes.c_int),
    "fp8mm_sf_from_canonical": ([_P, _I64, _I64, _P], ctypes.c_int),
    "fp8mm_workspace_bytes": ([_I64, _I64, _I64, ctypes.c_int32], ctypes.c_size_t),
    "fp8mm_pair_split_plan": ([_I64, _I64, _I64, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)], ctypes.c_int32),
    "fp8mm_quantize_gemm_workspace_bytes": ([_I64, _I64, _I64, ctypes.c_int32], ctypes.c_size_t),
    "fp8mm_status_str": ([ctypes.c_int], ctypes.c_char_p),
    "fp8mm_last_cuda_error": ([], ctypes.c_int),
    "fp8mm_last_device_error": ([], ctypes.c_uint),
    "fp8mm_selftest_wait_timeout": ([ctypes.c_uint32, _P], ctypes.c_int),
    "fp8mm_version": ([], ctypes.c_int),
}


def lib():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise Fp8mmError("load", -1, f"{LIB_PATH} is not built; run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(fn: str, status: int):
    if status != FP8MM_OK:
        raise Fp8mmError(fn, status, f"cuda error {lib().fp8mm_last_cuda_error()}")


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _u8(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t


def _need(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda or t.dtype != dtype:
        raise TypeError(f"{name}: expected a CUDA {dtype} tensor, got {t.dtype} on {t.device}")


def _ld(t: torch.Tensor, name: str) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name}: expected a 2-D tensor with unit column stride")
    return t.stride(0)


# ----------------------------------------------------------------- mode 1

def fp8_quantize_rowwise(x: torch.Tensor, q: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                         stream=None):
    """bf16 [rows, k] -> (E4M3 codes uint8 [rows, k], fp32 scale [rows])."""
    _need(x, torch.bfloat16, "x")
    rows, k = x.shape
    if q is None:
        q = torch.empty((rows, k), dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty((rows,), dtype=torch.float32, device=x.device)
    q = _u8(q)
    _check("fp8_quantize_rowwise", lib().fp8_quantize_rowwise(
        x.data_ptr(), rows, k, _ld(x, "x"), q.data_ptr(), _ld(q, "q"), scale.data_ptr(), _stream(stream)))
    return q, scale


def _ws_opts(workspace, kernel, small_m_ctas=0, flags=0):
    return Opts(workspace.data_ptr() if workspace is not None else None,
                workspace.numel() * workspace.element_size() if workspace is not None else 0,
                kernel, small_m_ctas, flags)


def fp8_gemm(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor, scale_b: torch.Tensor,
             c: torch.Tensor | None = None, kernel: int = KERNEL_AUTO, stream=None,
             workspace: torch.Tensor | None = None) -> torch.Tensor:
    """C bf16 [m, n] = diag(scale_a) (A x B^T) diag(scale_b); a [m,k], b [n,k] E4M3 codes.
    workspace (zeroed once, workspace_bytes(m, n, k) bytes): lets m > 64 shapes split the K range of the
    tiles of their last, partly filled wave of SM pairs over the pairs."""
    a, b = _u8(a), _u8(b)
    _need(a, torch.uint8, "a"); _need(b, torch.uint8, "b")
    _need(scale_a, torch.float32, "scale_a"); _need(scale_b, torch.float32, "scale_b")
    m, k = a.shape
    n = b.shape[0]
    if b.shape[1] != k or not (a.is_contiguous() and b.is_contiguous()):
        raise ValueError("a [m,k] and b [n,k] must be contiguous with the same k")
    if c is None:
        c = torch.empty((m, n), dtype=torch.bfloat16, device=a.device)
    opts = _ws_opts(workspace, kernel)
    _check("fp8_gemm", lib().fp8_gemm(a.data_ptr(), b.data_ptr(), m, n, k, scale_a.data_ptr(), scale_b.data_ptr(),
                                      c.data_ptr(), _ld(c, "c"), ctypes.byref(opts), _stream(stream)))
    return c


# ----------------------------------------------------------------- per tensor, FP8 out

def fp8_tensor_scale(x: torch.Tensor, scale: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bf16 [rows, k] -> fp32 [1] device scale = max|x| / 448 over the whole tensor (1 if all zero)."""
    _need(x, torch.bfloat16, "x")
    rows, k = x.shape
    if scale is None:
        scale = torch.empty((1,), dtype=torch.float32, device=x.device)
    _check("fp8_tensor_scale", lib().fp8_tensor_scale(x.data_ptr(), rows, k, _ld(x, "x") if k else k,
                                                      scale.data_ptr(), _stream(stream)))
    return scale


def fp8_quantize_static(x: torch.Tensor, scale: torch.Tensor, q: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """bf16 [rows, k] and a device fp32 scale -> E4M3 codes uint8 [rows, k] of x / scale."""
    _need(x, torch.bfloat16, "x"); _need(scale, torch.float32, "scale")
    rows, k = x.shape
    if q is None:
        q = torch.empty((rows, k), dtype=torch.uint8, device=x.device)
    q = _u8(q)
    _check("fp8_quantize_static", lib().fp8_quantize_static(x.data_ptr(), rows, k, _ld(x, "x"), scale.data_ptr(),
                                                            q.data_ptr(), _ld(q, "q"), _stream(stream)))
    return q


def fp8_gemm_e4m3_out(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor, scale_b: torch.Tensor,
                      scale_out: torch.Tensor, c: torch.Tensor | None = None, kernel: int = KERNEL_AUTO,
                      stream=None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """E4M3 codes uint8 [m, n] of diag(scale_a) (A x B^T) diag(scale_b) / scale_out (workspace as fp8_gemm)."""
    a, b = _u8(a), _u8(b)
    _need(a, torch.uint8, "a"); _need(b, torch.uint8, "b")
    _need(scale_a, torch.float32, "scale_a"); _need(scale_b, torch.float32, "scale_b")
    _need(scale_out, torch.float32, "scale_out")
    m, k = a.shape
    n = b.shape[0]
    if b.shape[1] != k or not (a.is_contiguous() and b.is_contiguous()):
        raise ValueError("a [m,k] and b [n,k] must be contiguous with the same k")
    if c is None:
        c = torch.empty((m, n), dtype=torch.uint8, device=a.device)
    c = _u8(c)
    opts = _ws_opts(workspace, kernel)
    _check("fp8_gemm_e4m3_out", lib().fp8_gemm_e4m3_out(
        a.data_ptr(), b.data_ptr(), m, n, k, scale_a.data_ptr(), scale_b.data_ptr(), scale_out.data_ptr(),
        c.data_ptr(), _ld(c, "c"), ctypes.byref(opts), _stream(stream)))
    return c


# ----------------------------------------------------------------- mode 2

def sf_bytes(rows: int, k: int) -> int:
    return int(lib().fp8mm_sf_bytes(rows, k))


def sf_offset(rows: int, k: int, row: int, block: int) -> int:
    return int(lib().fp8mm_sf_offset(rows, k, row, block))


def sf_to_canonical(sf: torch.Tensor, rows: int, k: int) -> torch.Tensor:
    """Library scale layout (CPU uint8 tensor) -> canonical [rows, k/32] (CPU)."""
    src = sf.detach().cpu().contiguous()
    out = torch.empty((rows, k // 32), dtype=torch.uint8)
    _check("fp8mm_sf_to_canonical", lib().fp8mm_sf_to_canonical(src.data_ptr(), rows, k, out.data_ptr()))
    return out


def sf_from_canonical(canonical: torch.Tensor, rows: int, k: int) -> torch.Tensor:
    """Canonical [rows, k/32] (CPU uint8) -> library scale layout (CPU)."""
    src = canonical.detach().cpu().contiguous()
    out = torch.empty((sf_bytes(rows, k),), dtype=torch.uint8)
    _check("fp8mm_sf_from_canonical", lib().fp8mm_sf_from_canonical(src.data_ptr(), rows, k, out.data_ptr()))
    return out


def mxfp8_quantize(x: torch.Tensor, q: torch.Tensor | None = None, sf: torch.Tensor | None = None, stream=None):
    """bf16 [rows, k] -> (E4M3 codes uint8 [rows, k], scales uint8 [sf_bytes] in the library layout)."""
    _need(x, torch.bfloat16, "x")
    rows, k = x.shape
    if q is None:
        q = torch.empty((rows, k), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty((max(sf_bytes(rows, k), 1),), dtype=torch.uint8, device=x.device)
    q = _u8(q)
    _check("mxfp8_quantize", lib().mxfp8_quantize(x.data_ptr(), rows, k, _ld(x, "x"), q.data_ptr(), _ld(q, "q"),
                                                  sf.data_ptr(), _stream(stream)))
    return q, sf


def sf8x4_bytes(rows: int, k: int) -> int:
    return int(lib().fp8mm_sf8x4_bytes(rows, k))


def sf8x4_offset(rows: int, k: int, row: int, block: int) -> int:
    return int(lib().fp8mm_sf8x4_offset(rows, k, row, block))


def mxfp8_quantize_8x4(x: torch.Tensor, q: torch.Tensor | None = None, sf: torch.Tensor | None = None,
                       stream=None):
    """mxfp8_quantize with the scales in the small-M (8x4) layout: (codes uint8 [rows, k],
    scales uint8 [sf8x4_bytes]); for activations of a few token rows fed to mxfp8_gemm(sf_a_8x4=True)."""
    _need(x, torch.bfloat16, "x")
    rows, k = x.shape
    if q is None:
        q = torch.empty((rows, k), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty((max(sf8x4_bytes(rows, k), 1),), dtype=torch.uint8, device=x.device)
    q = _u8(q)
    _check("mxfp8_quantize_8x4", lib().mxfp8_quantize_8x4(x.data_ptr(), rows, k, _ld(x, "x"), q.data_ptr(),
                                                          _ld(q, "q"), sf.data_ptr(), _stream(stream)))
    return q, sf


def workspace_bytes(m: int, n: int, k: int, ctas: int = 0) -> int:
    return int(lib().fp8mm_workspace_bytes(m, n, k, ctas))


def pair_split_plan(m: int, n: int, k: int, pairs: int) -> tuple[int, int]:
    """(K parts per split tile, tiles run whole) of the paired kernel's split with `pairs` SM pairs."""
    dp = ctypes.c_int32(0)
    split = int(lib().fp8mm_pair_split_plan(m, n, k, pairs, ctypes.byref(dp)))
    return split, int(dp.value)


def quantize_gemm_workspace_bytes(m: int, n: int, k: int, ctas: int = 0) -> int:
    return int(lib().fp8mm_quantize_gemm_workspace_bytes(m, n, k, ctas))


def mxfp8_gemm(a: torch.Tensor, sf_a: torch.Tensor, b: torch.Tensor, sf_b: torch.Tensor,
               c: torch.Tensor | None = None, workspace: torch.Tensor | None = None, kernel: int = KERNEL_AUTO,
               small_m_ctas: int = 0, weights_ready: bool = False, stream=None,
               split_via_workspace: bool = False, sf_a_8x4: bool = False) -> torch.Tensor:
    """C bf16 [m, n] = block-scaled A x B^T; a [m,k], b [n,k] codes with their library-layout scales.
    workspace (zeroed once, workspace_bytes(m, n, k, small_m_ctas) bytes): the small-M kernel's stream-K
    split for m <= 64 where the CTA count is not tile-aligned (aligned splits reduce inside clusters);
    for m > 64 the K split of the tiles of the last, partly filled wave of SM pairs.
    weights_ready: b and sf_b were complete before the preceding kernel on the stream started (see
    FP8MM_FLAG_WEIGHTS_READY).  split_via_workspace: FP8MM_FLAG_SPLIT_VIA_WORKSPACE.  sf_a_8x4: sf_a is in
    the small-M layout of mxfp8_quantize_8x4 (m <= 64 only)."""
    a, b = _u8(a), _u8(b)
    _need(a, torch.uint8, "a"); _need(b, torch.uint8, "b")
    _need(sf_a, torch.uint8, "sf_a"); _need(sf_b, torch.uint8, "sf_b")
    m, k = a.shape
    n = b.shape[0]
    if b.shape[1] != k or not (a.is_contiguous() and b.is_contiguous()):
        raise ValueError("a [m,k] and b [n,k] must be contiguous with the same k")
    if c is None:
        c = torch.empty((m, n), dtype=torch.bfloat16, device=a.device)
    flags = ((FLAG_WEIGHTS_READY if weights_ready else 0) | (FLAG_SPLIT_VIA_WORKSPACE if split_via_workspace else 0)
             | (FLAG_SF_A_8X4 if sf_a_8x4 else 0))
    opts = _ws_opts(workspace, kernel, small_m_ctas, flags)
    _check("mxfp8_gemm", lib().mxfp8_gemm(a.data_ptr(), sf_a.data_ptr(), b.data_ptr(), sf_b.data_ptr(), m, n, k,
                                          c.data_ptr(), _ld(c, "c"), ctypes.byref(opts), _stream(stream)))
    return c


def mxfp8_quantize_gemm(a: torch.Tensor, b: torch.Tensor, sf_b: torch.Tensor, c: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None, kernel: int = KERNEL_AUTO, small_m_ctas: int = 0,
                        weights_ready: bool = False, stream=None, split_via_workspace: bool = False) -> torch.Tensor:
    """C bf16 [m, n] = mxfp8_gemm(mxfp8_quantize(a), b) for m <= 64 from the bf16 activation a [m, k]:
    quantized inside the GEMM kernel for m <= 8, else by its own launch into the workspace tail
    (workspace of quantize_gemm_workspace_bytes(m, n, k, small_m_ctas) bytes, required for m > 8)."""
    b = _u8(b)
    _need(a, torch.bfloat16, "a"); _need(b, torch.uint8, "b"); _need(sf_b, torch.uint8, "sf_b")
    m, k = a.shape
    n = b.shape[0]
    if b.shape[1] != k or not b.is_contiguous():
        raise ValueError("b [n,k] must be contiguous with the k of a")
    if c is None:
        c = torch.empty((m, n), dtype=torch.bfloat16, device=a.device)
    opts = Opts(workspace.data_ptr() if workspace is not None else None,
                workspace.numel() * workspace.element_size() if workspace is not None else 0,
                kernel, small_m_ctas,
                (FLAG_WEIGHTS_READY if weights_ready else 0) | (FLAG_SPLIT_VIA_WORKSPACE if split_via_workspace else 0))
    _check("mxfp8_quantize_gemm", lib().mxfp8_quantize_gemm(
        a.data_ptr(), _ld(a, "a"), b.data_ptr(), sf_b.data_ptr(), m, n, k, c.data_ptr(), _ld(c, "c"),
        ctypes.byref(opts), _stream(stream)))
    return c


# ----------------------------------------------------------------- KV cache

def concat_mla_k(k_nope: torch.Tensor, k_rope: torch.Tensor, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """k_nope [T, H, nope], k_rope [T, H or 1, rope] (1 = one rope vector per token for all heads)
    -> out [T, H, nope + rope]; 1-byte (float8 / uint8) or 2-byte elements, any 16-byte-aligned strides."""
    if k_nope.dim() != 3 or k_rope.dim() != 3 or not k_nope.is_cuda or not k_rope.is_cuda:
        raise ValueError("k_nope and k_rope must be 3-D CUDA tensors")
    if k_nope.element_size() != k_rope.element_size() or k_nope.dtype != k_rope.dtype:
        raise TypeError("k_nope and k_rope must have the same dtype")
    T, H, dn = k_nope.shape
    dr = k_rope.shape[2]
    if k_rope.shape[0] != T or k_rope.shape[1] not in (1, H) or k_nope.stride(2) != 1 or k_rope.stride(2) != 1:
        raise ValueError("k_rope must be [T, H or 1, rope] with unit element stride, k_nope unit element stride")
    if out is None:
        out = torch.empty((T, H, dn + dr), dtype=k_nope.dtype, device=k_nope.device)
    if out.shape != (T, H, dn + dr) or out.stride(2) != 1 or out.dtype != k_nope.dtype:
        raise ValueError("out must be [T, H, nope + rope] of the input dtype with unit element stride")
    rope_sh = 0 if k_rope.shape[1] == 1 else k_rope.stride(1)
    _check("concat_mla_k", lib().concat_mla_k(
        k_nope.data_ptr(), k_rope.data_ptr(), out.data_ptr(), T, H, dn, dr, k_nope.element_size(),
        k_nope.stride(0), k_nope.stride(1), k_rope.stride(0), rope_sh, out.stride(0), out.stride(1),
        _stream(stream)))
    return out


# ----------------------------------------------------------------- misc

def last_device_error() -> int:
    return int(lib().fp8mm_last_device_error())


def selftest_wait_timeout(timeout_us: int = 2000, stream=None) -> int:
    return int(lib().fp8mm_selftest_wait_timeout(timeout_us, _stream(stream)))


def version() -> int:
    return int(lib().fp8mm_version())
