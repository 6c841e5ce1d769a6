"""CPU oracle for the scaled FP8 / MXFP8 GEMM and its quantizers (ctypes over
``liboracle.so``, built from ``oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import this package.  The
product library never calls it and shares no code with it.

Every function takes and returns numpy arrays.  bf16 inputs are passed as their
uint16 bit patterns (``torch_bf16.view(torch.int16).numpy().view(np.uint16)``).
The arithmetic and its citations are in ``oracle.h`` / ``oracle.c``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_encode.argtypes = [ctypes.c_double]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_mx_exponent.argtypes = [ctypes.c_double]
        L.orc_mx_exponent.restype = ctypes.c_int
        L.orc_quantize_rowwise.argtypes = [P, I64, I64, I64, P, I64, P, ctypes.c_int]
        L.orc_quantize_rowwise.restype = None
        L.orc_tensor_scale.argtypes = [P, I64, I64, I64]
        L.orc_tensor_scale.restype = ctypes.c_float
        L.orc_quantize_static.argtypes = [P, I64, I64, I64, ctypes.c_float, P, I64, ctypes.c_int]
        L.orc_quantize_static.restype = None
        L.orc_mx_quantize.argtypes = [P, I64, I64, I64, P, I64, P, ctypes.c_int]
        L.orc_mx_quantize.restype = None
        L.orc_gemm_rowwise.argtypes = [P, P, I64, I64, I64, P, P, P, P, ctypes.c_int]
        L.orc_gemm_rowwise.restype = None
        L.orc_gemm_mx.argtypes = [P, P, P, P, I64, I64, I64, P, P, ctypes.c_int]
        L.orc_gemm_mx.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def e4m3_decode_table() -> np.ndarray:
    """float64[256]: the value of every E4M3 code (NaN for 0x7F and 0xFF)."""
    L = lib()
    return np.array([L.orc_e4m3_decode(v) for v in range(256)], dtype=np.float64)


def e4m3_encode(values) -> np.ndarray:
    """uint8 codes of finite float64 values (RNE, saturating, sign kept)."""
    L = lib()
    v = np.asarray(values, dtype=np.float64)
    return np.array([L.orc_e4m3_encode(float(x)) for x in v.ravel()],
                    dtype=np.uint8).reshape(v.shape)


def mx_exponent(amax) -> np.ndarray:
    """int32 UE8M0 exponent of each block maximum (ceil(log2(a/448))+127)."""
    L = lib()
    a = np.asarray(amax, dtype=np.float64)
    return np.array([L.orc_mx_exponent(float(x)) for x in a.ravel()],
                    dtype=np.int32).reshape(a.shape)


def quantize_rowwise(x_bits: np.ndarray, nthreads: int = 0):
    """Mode-1 quantizer.  x_bits: uint16 [R, K] bf16 patterns.
    Returns (q uint8 [R, K], s float32 [R])."""
    x = _c(x_bits, np.uint16)
    R, K = x.shape
    q = np.empty((R, K), dtype=np.uint8)
    s = np.empty((R,), dtype=np.float32)
    lib().orc_quantize_rowwise(_ptr(x), R, K, K, _ptr(q), K, _ptr(s),
                               nthreads or default_threads())
    return q, s


def tensor_scale(x_bits: np.ndarray) -> np.float32:
    """Per-tensor scale fp32(max|x| / 448) (1 for an all-zero tensor)."""
    x = _c(x_bits, np.uint16)
    rows, k = x.shape
    return np.float32(lib().orc_tensor_scale(_ptr(x), rows, k, k))


def quantize_static(x_bits: np.ndarray, scale, nthreads: int = 0) -> np.ndarray:
    """E4M3 codes of fp32(x / scale) for one given fp32 scale."""
    x = _c(x_bits, np.uint16)
    rows, k = x.shape
    q = np.empty((rows, k), dtype=np.uint8)
    lib().orc_quantize_static(_ptr(x), rows, k, k, ctypes.c_float(float(np.float32(scale))), _ptr(q), k,
                              nthreads or default_threads())
    return q


def concat_mla_k(k_nope: np.ndarray, k_rope: np.ndarray) -> np.ndarray:
    """Key assembly of page "[flashinfer] FlashInfer, FP8 지원으로 장문 컨텍스트 추론
    성능을 극적으로 향상시키다" (코드 분석 items 1 and 3): for every token t and head h,
    the nope part of the key followed by its rope part; a k_rope with one head is the
    same rope vector for every head.  Inputs [T, H, nope] and [T, H or 1, rope] of any
    element type; the output [T, H, nope + rope] holds the input elements unchanged."""
    T, H, _ = k_nope.shape
    rope = np.broadcast_to(k_rope, (T, H, k_rope.shape[2]))
    return np.concatenate([k_nope, rope], axis=2)


def mx_quantize(x_bits: np.ndarray, nthreads: int = 0):
    """Mode-2 quantizer.  x_bits: uint16 [R, K] bf16 patterns, K % 32 == 0.
    Returns (q uint8 [R, K], sf uint8 [R, K/32] canonical row-major)."""
    x = _c(x_bits, np.uint16)
    R, K = x.shape
    assert K % 32 == 0
    q = np.empty((R, K), dtype=np.uint8)
    sf = np.empty((R, K // 32), dtype=np.uint8)
    lib().orc_mx_quantize(_ptr(x), R, K, K, _ptr(q), K, _ptr(sf),
                          nthreads or default_threads())
    return q, sf


def gemm_rowwise(qa, qb, sa, sb, nthreads: int = 0, want_bound: bool = True):
    """Mode-1 reference.  qa uint8 [M,K], qb uint8 [N,K] (B^T), sa f32 [M],
    sb f32 [N].  Returns (c_ref f64 [M,N], bound f64 [M,N] or None)."""
    qa = _c(qa, np.uint8); qb = _c(qb, np.uint8)
    sa = _c(sa, np.float32); sb = _c(sb, np.float32)
    M, K = qa.shape
    N = qb.shape[0]
    assert qb.shape[1] == K and sa.shape == (M,) and sb.shape == (N,)
    c = np.empty((M, N), dtype=np.float64)
    b = np.empty((M, N), dtype=np.float64) if want_bound else None
    lib().orc_gemm_rowwise(_ptr(qa), _ptr(qb), M, N, K, _ptr(sa), _ptr(sb), _ptr(c),
                           _ptr(b) if b is not None else None,
                           nthreads or default_threads())
    return c, b


def gemm_mx(qa, sfa, qb, sfb, nthreads: int = 0, want_bound: bool = True):
    """Mode-2 reference.  qa uint8 [M,K], sfa uint8 [M,K/32], qb uint8 [N,K],
    sfb uint8 [N,K/32] (canonical).  Returns (c_ref, bound)."""
    qa = _c(qa, np.uint8); qb = _c(qb, np.uint8)
    sfa = _c(sfa, np.uint8); sfb = _c(sfb, np.uint8)
    M, K = qa.shape
    N = qb.shape[0]
    assert K % 32 == 0 and qb.shape[1] == K
    assert sfa.shape == (M, K // 32) and sfb.shape == (N, K // 32)
    c = np.empty((M, N), dtype=np.float64)
    b = np.empty((M, N), dtype=np.float64) if want_bound else None
    lib().orc_gemm_mx(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), M, N, K, _ptr(c),
                      _ptr(b) if b is not None else None, nthreads or default_threads())
    return c, b
