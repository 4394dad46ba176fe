"""ctypes front-end of the fp64 CPU oracle (oracle/oracle.c).

TEST INFRASTRUCTURE ONLY: tests, the smoke check and the benchmark's CPU
baseline call this module; the product path (libbi.so and its binding) never
does.  Arguments are numpy arrays: bf16 tensors as ``uint16`` bit patterns,
fp32 tensors as ``float32``.  Results come back as ``float64`` arrays.

Each wrapper names the definition it evaluates; the C source carries the
citations of the pages.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None
_i64 = ctypes.c_int64
_ptr = ctypes.c_void_p


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        for name in ("oracle_matmul", "oracle_addmm", "oracle_rmsnorm", "oracle_mean_f32",
                     "oracle_log_softmax_f32", "oracle_log_softmax_bf16", "oracle_silu_mul",
                     "oracle_silu_mul_f64"):
            getattr(lib, name).restype = ctypes.c_int
        lib.oracle_matmul.argtypes = [_ptr, _i64, _ptr, _i64, ctypes.c_int, _ptr, _i64,
                                      _i64, _i64, _i64, ctypes.c_int]
        lib.oracle_addmm.argtypes = [_ptr, _i64, _ptr, _i64, _ptr, _i64, ctypes.c_int, _ptr, _i64,
                                     _i64, _i64, _i64, ctypes.c_int]
        lib.oracle_rmsnorm.argtypes = [_ptr, _ptr, _ptr, _i64, _i64, ctypes.c_double, ctypes.c_int]
        lib.oracle_mean_f32.argtypes = [_ptr, _ptr, _i64, _i64, ctypes.c_int]
        lib.oracle_log_softmax_f32.argtypes = [_ptr, _ptr, _i64, _i64, ctypes.c_int]
        lib.oracle_log_softmax_bf16.argtypes = [_ptr, _ptr, _i64, _i64, ctypes.c_int]
        lib.oracle_silu_mul.argtypes = [_ptr, _ptr, _i64, _i64, ctypes.c_int]
        lib.oracle_silu_mul_f64.argtypes = [_ptr, _ptr, _i64, _i64, ctypes.c_int]
        lib.oracle_decode_attention.restype = ctypes.c_int
        lib.oracle_decode_attention.argtypes = [_ptr, _ptr, _ptr, _ptr, _ptr, _i64, _i64, _i64, _i64, _i64,
                                                ctypes.c_double, ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def max_threads() -> int:
    return int(_lib().oracle_max_threads())


def _threads(nthreads):
    return int(nthreads) if nthreads else (os.cpu_count() or 1)


def _as(a, dtype, name):
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError(f"{name}: expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def _rowmajor_ld(a, name):
    """Leading dimension (elements) of a 2-D array whose rows are unit-stride."""
    if a.ndim != 2:
        raise ValueError(f"{name}: expected a 2-D array")
    if a.size == 0:
        return max(a.shape[1], 1)
    if a.shape[1] > 1 and a.strides[1] != a.itemsize:
        raise ValueError(f"{name}: rows must be unit-stride")
    if a.shape[0] > 1:
        if a.strides[0] % a.itemsize:
            raise ValueError(f"{name}: row stride is not a whole number of elements")
        return a.strides[0] // a.itemsize
    return max(a.shape[1], 1)


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments")


def matmul(a_bits, b_bits, b_layout: str = "kn", nthreads=None) -> np.ndarray:
    """C = A.B in binary64 (torch.mm).  b_layout 'kn': B is [K, N]; 'nk': B is [N, K]."""
    a = _as(a_bits, np.uint16, "A")
    b = _as(b_bits, np.uint16, "B")
    lay = {"kn": 0, "nk": 1}[b_layout]
    M, K = a.shape
    N = b.shape[1] if lay == 0 else b.shape[0]
    kb = b.shape[0] if lay == 0 else b.shape[1]
    if kb != K:
        raise ValueError("inner dimensions differ")
    c = np.zeros((M, N), dtype=np.float64)
    rc = _lib().oracle_matmul(a.ctypes.data, _rowmajor_ld(a, "A"), b.ctypes.data,
                              _rowmajor_ld(b, "B"), lay, c.ctypes.data, max(N, 1), M, N, K,
                              _threads(nthreads))
    _check(rc, "oracle_matmul")
    return c


def addmm(input_bits, a_bits, b_bits, b_layout: str = "kn", nthreads=None) -> np.ndarray:
    """C = input + A.B (torch.addmm, alpha = beta = 1); input is a bias [N] or a matrix [M, N]."""
    inp = _as(input_bits, np.uint16, "input")
    a = _as(a_bits, np.uint16, "A")
    b = _as(b_bits, np.uint16, "B")
    lay = {"kn": 0, "nk": 1}[b_layout]
    M, K = a.shape
    N = b.shape[1] if lay == 0 else b.shape[0]
    if inp.ndim == 1:
        if inp.shape[0] != N:
            raise ValueError("bias length differs from N")
        ld_in = 0
    else:
        if inp.shape != (M, N):
            raise ValueError("input shape differs from [M, N]")
        ld_in = _rowmajor_ld(inp, "input")
    c = np.zeros((M, N), dtype=np.float64)
    rc = _lib().oracle_addmm(inp.ctypes.data, ld_in, a.ctypes.data, _rowmajor_ld(a, "A"),
                             b.ctypes.data, _rowmajor_ld(b, "B"), lay, c.ctypes.data, max(N, 1),
                             M, N, K, _threads(nthreads))
    _check(rc, "oracle_addmm")
    return c


def rmsnorm(x_bits, w_bits, eps: float, nthreads=None) -> np.ndarray:
    """y = x * (1 / sqrt(mean(x^2) + eps)) * w over the last dimension."""
    x = np.ascontiguousarray(_as(x_bits, np.uint16, "x"))
    w = np.ascontiguousarray(_as(w_bits, np.uint16, "w"))
    M, H = x.shape
    if w.shape != (H,):
        raise ValueError("weight length differs from H")
    y = np.zeros((M, H), dtype=np.float64)
    _check(_lib().oracle_rmsnorm(x.ctypes.data, w.ctypes.data, y.ctypes.data, M, H, float(eps),
                                 _threads(nthreads)), "oracle_rmsnorm")
    return y


def mean(x, nthreads=None) -> np.ndarray:
    """y_i = sum_j x_ij / H for fp32 x [M, H]."""
    x = np.ascontiguousarray(_as(x, np.float32, "x"))
    M, H = x.shape
    y = np.zeros((M,), dtype=np.float64)
    _check(_lib().oracle_mean_f32(x.ctypes.data, y.ctypes.data, M, H, _threads(nthreads)),
           "oracle_mean_f32")
    return y


def log_softmax(x, nthreads=None) -> np.ndarray:
    """y = (x - max) - log(sum exp(x - max)) per row; x is fp32 or bf16 bits (uint16)."""
    x = np.ascontiguousarray(np.asarray(x))
    M, V = x.shape
    y = np.zeros((M, V), dtype=np.float64)
    if x.dtype == np.float32:
        rc = _lib().oracle_log_softmax_f32(x.ctypes.data, y.ctypes.data, M, V, _threads(nthreads))
    elif x.dtype == np.uint16:
        rc = _lib().oracle_log_softmax_bf16(x.ctypes.data, y.ctypes.data, M, V, _threads(nthreads))
    else:
        raise TypeError("x must be float32 or bf16 bits (uint16)")
    _check(rc, "oracle_log_softmax")
    return y


def silu_mul(gu_bits, nthreads=None) -> np.ndarray:
    """h = silu(gate) * up where gate = gu[:, :F] and up = gu[:, F:]."""
    gu = np.ascontiguousarray(_as(gu_bits, np.uint16, "gu"))
    M, F2 = gu.shape
    if F2 % 2:
        raise ValueError("gu must have an even number of columns")
    F = F2 // 2
    h = np.zeros((M, F), dtype=np.float64)
    _check(_lib().oracle_silu_mul(gu.ctypes.data, h.ctypes.data, M, F, _threads(nthreads)),
           "oracle_silu_mul")
    return h


def silu_mul_f64(gu, nthreads=None) -> np.ndarray:
    """h = silu(gate) * up on binary64 gate|up columns (no rounding in between)."""
    gu = np.ascontiguousarray(_as(gu, np.float64, "gu"))
    M, F2 = gu.shape
    if F2 % 2:
        raise ValueError("gu must have an even number of columns")
    F = F2 // 2
    h = np.zeros((M, F), dtype=np.float64)
    _check(_lib().oracle_silu_mul_f64(gu.ctypes.data, h.ctypes.data, M, F, _threads(nthreads)),
           "oracle_silu_mul_f64")
    return h


def matmul_silu_mul(a_bits, b_bits, b_layout: str = "nk", nthreads=None) -> np.ndarray:
    """silu(A . gate) * (A . up) with B = [gate; up] (2F outputs), all in binary64."""
    return silu_mul_f64(matmul(a_bits, b_bits, b_layout, nthreads), nthreads)


def decode_attention(q_bits, k_bits, v_bits, lens, scale: float, nthreads=None) -> np.ndarray:
    """Softmax attention of one query token per sequence over its first lens[b] cached tokens.
    q [B, Hq, D], k and v [B, Lmax, Hkv, D] as bf16 bits; query head h reads kv head h // (Hq/Hkv)."""
    q = np.ascontiguousarray(_as(q_bits, np.uint16, "q"))
    k = np.ascontiguousarray(_as(k_bits, np.uint16, "k"))
    v = np.ascontiguousarray(_as(v_bits, np.uint16, "v"))
    lens = np.ascontiguousarray(np.asarray(lens, dtype=np.int32))
    B, Hq, D = q.shape
    Bk, Lmax, Hkv, Dk = k.shape
    if Bk != B or Dk != D or v.shape != k.shape or lens.shape != (B,):
        raise ValueError("shape mismatch")
    o = np.zeros((B, Hq, D), dtype=np.float64)
    _check(_lib().oracle_decode_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, lens.ctypes.data,
                                          o.ctypes.data, B, Hq, Hkv, D, Lmax, float(scale),
                                          _threads(nthreads)), "oracle_decode_attention")
    return o

