"""ctypes view of ``ordered.c`` (fixed-order float32 / sequential float64).

Test infrastructure only (see the package docstring). The shared object is
built next to the source by :func:`build` (gcc, no CUDA).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ordered.c")
_LIB = os.path.join(_HERE, "libordered.so")
_lib = None

_CFLAGS = ["-O2", "-std=gnu99", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-fopenmp"]


def build(force: bool = False) -> str:
    """Compile ordered.c into libordered.so (plain C, gcc)."""
    if force or not os.path.exists(_LIB) or \
            os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", _LIB, "-lm"])
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        i64, f32, f64 = ctypes.c_int64, ctypes.c_float, ctypes.c_double
        p = ctypes.c_void_p
        _lib.seq_sum_f64.restype = f64
        _lib.seq_sum_f64.argtypes = [p, i64]
        _lib.seq_sum_rows_f64.argtypes = [p, i64, i64, p]
        _lib.mixed_sum_rows_f64.argtypes = [p, p, i64, i64, p]
        _lib.seq_sum_f32.restype = f32
        _lib.seq_sum_f32.argtypes = [p, i64]
        _lib.grouped_sum_f32.restype = f32
        _lib.grouped_sum_f32.argtypes = [p, i64, i64]
        _lib.rmsnorm_f32.argtypes = [p, p, p, i64, i64, f32]
        _lib.gemm_f32.argtypes = [p, p, p, i64, i64, i64]
        _lib.attention_f32.argtypes = [p, p, p, p, i64, i64, i64, i64, i64,
                                       f32, p, p, i64]
        _lib.ordered_set_threads.argtypes = [ctypes.c_int]
        _lib.ordered_max_threads.restype = ctypes.c_int
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def seq_sum_f64(v) -> float:
    v = _c(v, np.float64)
    return lib().seq_sum_f64(_ptr(v), v.size)


def seq_sum_rows_f64(v) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape[0], np.float64)
    lib().seq_sum_rows_f64(_ptr(v), v.shape[0], v.shape[1], _ptr(out))
    return out


def mixed_sum_rows_f64(v, is_int) -> np.ndarray:
    """Row sums with CPython's built-in sum() semantics for mixed int/float
    lists (see mixed_sum_f64 in ordered.c)."""
    v = _c(v, np.float64)
    f = _c(is_int, np.int8)
    out = np.empty(v.shape[0], np.float64)
    lib().mixed_sum_rows_f64(_ptr(v), _ptr(f), v.shape[0], v.shape[1], _ptr(out))
    return out


def seq_sum_f32(v) -> np.float32:
    v = _c(v, np.float32)
    return np.float32(lib().seq_sum_f32(_ptr(v), v.size))


def grouped_sum_f32(v, group: int) -> np.float32:
    v = _c(v, np.float32)
    return np.float32(lib().grouped_sum_f32(_ptr(v), v.size, group))


def rmsnorm_f32(x, gamma, eps: float) -> np.ndarray:
    x = _c(x, np.float32)
    g = _c(gamma, np.float32)
    y = np.empty_like(x)
    lib().rmsnorm_f32(_ptr(x), _ptr(g), _ptr(y), x.shape[0], x.shape[1], eps)
    return y


def gemm_f32(A, W) -> np.ndarray:
    """C = A W^T, float32, fmaf left to right over k."""
    A = _c(A, np.float32)
    W = _c(W, np.float32)
    C = np.empty((A.shape[0], W.shape[0]), np.float32)
    lib().gemm_f32(_ptr(A), _ptr(W), _ptr(C), A.shape[0], W.shape[0], A.shape[1])
    return C


def set_threads(n: int) -> None:
    """OpenMP threads of the parallel loops (timing only; results do not
    depend on it)."""
    lib().ordered_set_threads(int(n))


def max_threads() -> int:
    return int(lib().ordered_max_threads())


def attention_f32(q, k, v, q_pos, scale: float, threads: int | None = None) -> np.ndarray:
    q = _c(q, np.float32)
    k = _c(k, np.float32)
    v = _c(v, np.float32)
    pos = _c(q_pos, np.int32)
    n, hq, d = q.shape
    L, hkv, _ = k.shape
    if threads is None:
        threads = max(1, os.cpu_count() or 1)
    scratch = np.empty((threads, max(L, 1)), np.float32)
    out = np.empty_like(q)
    lib().attention_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(pos), n, L, hq, hkv, d,
                        scale, _ptr(out), _ptr(scratch), threads)
    return out
