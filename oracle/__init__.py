"""CPU oracle for the batched exact Lloyd iteration (numpy front end to km_oracle.cpp).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may import this package; the CUDA library never does.

Every function restates the method as the Flash-KMeans pages define it
(papernotes.org "Flash-KMeans: Fast and Memory-Efficient Exact K-Means",
方法详解: 整体框架, 关键设计 1 and 2), in double precision; see km_oracle.cpp
for the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, F16 = 0, 1
_P = ctypes.c_void_p
_I = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile liboracle.so (plain C++17, std::thread)."""
    src = os.path.join(_HERE, "km_oracle.cpp")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["g++", "-std=c++17", "-O2", "-shared", "-fPIC", "-pthread", "-o", _SO, src])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.oracle_hw_threads.restype = ctypes.c_int
        lib.oracle_f16_decode.argtypes = [_P, _P, _I]
        lib.oracle_f16_encode.argtypes = [_P, _P, _I]
        lib.oracle_round_centroids.argtypes = [_P, ctypes.c_int, _I, _P]
        lib.oracle_assign.restype = ctypes.c_int
        lib.oracle_assign.argtypes = [_P, ctypes.c_int, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P, ctypes.c_int]
        lib.oracle_sort.restype = ctypes.c_int
        lib.oracle_sort.argtypes = [_P, _I, _I, _I, _P, _P, _P]
        lib.oracle_update.restype = ctypes.c_int
        lib.oracle_update.argtypes = [_P, ctypes.c_int, _P, _I, _I, _I, _I, _P, _P, _P, _P, ctypes.c_int]
        lib.oracle_cost.restype = ctypes.c_int
        lib.oracle_cost.argtypes = [_P, ctypes.c_int, _P, _P, _I, _I, _I, _I, _P]
        lib.oracle_lloyd.restype = ctypes.c_int
        lib.oracle_lloyd.argtypes = [_P, ctypes.c_int, _P, _I, _I, _I, _I, ctypes.c_int, _P, _P, _P, ctypes.c_int]
        lib.oracle_lloyd_tol.restype = ctypes.c_int
        lib.oracle_lloyd_tol.argtypes = [_P, ctypes.c_int, _P, _I, _I, _I, _I, ctypes.c_int, ctypes.c_double, _P, _P,
                                         _P, _P, _P, ctypes.c_int]
        _lib = lib
    return _lib


def threads() -> int:
    return max(1, int(_load().oracle_hw_threads()))


def _dtype_code(X: np.ndarray) -> int:
    if X.dtype == np.float16:
        return F16
    if X.dtype == np.float32:
        return F32
    raise TypeError(f"X must be float16 or float32, got {X.dtype}")


def _c(a: np.ndarray, dtype=None) -> np.ndarray:
    a = np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))
    return a


def f16_decode(bits: np.ndarray) -> np.ndarray:
    bits = _c(bits, np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().oracle_f16_decode(bits.ctypes.data, out.ctypes.data, bits.size)
    return out


def f16_encode(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_f16_encode(x.ctypes.data, out.ctypes.data, x.size)
    return out


def round_centroids(C: np.ndarray, dtype_code: int) -> np.ndarray:
    """fp32 centroids as the assignment sees them (rounded to X's dtype), in float64."""
    C = _c(C, np.float32)
    out = np.empty(C.shape, dtype=np.float64)
    _load().oracle_round_centroids(C.ctypes.data, dtype_code, C.size, out.ctypes.data)
    return out


def assign(X: np.ndarray, C: np.ndarray, rows: np.ndarray | None = None, nthreads: int | None = None,
           chat: np.ndarray | None = None):
    """Nearest centroid per point.  X [B,N,d] (fp16/fp32), C [B,K,d] fp32.

    Returns (labels, d1, d2): for the selected flattened rows b*N+i (all rows if
    rows is None), the lowest-index argmin, the minimum squared distance and the
    second smallest one (+inf when K == 1).
    """
    X = _c(X)
    B, N, d = X.shape
    K = C.shape[1]
    code = _dtype_code(X)
    if chat is None:
        chat = round_centroids(C, code)
    n = B * N if rows is None else len(rows)
    rows_a = None if rows is None else _c(rows, np.int64)
    labels = np.empty(n, dtype=np.int32)
    d1 = np.empty(n, dtype=np.float64)
    d2 = np.empty(n, dtype=np.float64)
    rc = _load().oracle_assign(X.ctypes.data, code, chat.ctypes.data, B, N, K, d,
                               None if rows_a is None else rows_a.ctypes.data, n,
                               labels.ctypes.data, d1.ctypes.data, d2.ctypes.data, nthreads or threads())
    if rc:
        raise ValueError(f"oracle_assign failed ({rc})")
    if rows is None:
        return labels.reshape(B, N), d1.reshape(B, N), d2.reshape(B, N)
    return labels, d1, d2


def sort_labels(labels: np.ndarray, K: int):
    """Stable argsort per batch: (sorted_idx [B,N], counts [B,K], offsets [B,K+1])."""
    labels = _c(labels, np.int32)
    B, N = labels.shape
    sidx = np.empty((B, N), dtype=np.int32)
    counts = np.empty((B, K), dtype=np.int32)
    offsets = np.empty((B, K + 1), dtype=np.int32)
    rc = _load().oracle_sort(labels.ctypes.data, B, N, K, sidx.ctypes.data, counts.ctypes.data,
                             offsets.ctypes.data)
    if rc:
        raise ValueError(f"oracle_sort failed ({rc}): labels out of [0, K)")
    return sidx, counts, offsets


def update(X: np.ndarray, labels: np.ndarray, C_prev: np.ndarray, nthreads: int | None = None):
    """New centroids from a labelling: (C_out fp32 [B,K,d], sums float64 [B,K,d], counts int32 [B,K])."""
    X = _c(X)
    B, N, d = X.shape
    K = C_prev.shape[1]
    labels = _c(labels, np.int32)
    C_prev = _c(C_prev, np.float32)
    C_out = np.empty_like(C_prev)
    sums = np.empty((B, K, d), dtype=np.float64)
    counts = np.empty((B, K), dtype=np.int32)
    rc = _load().oracle_update(X.ctypes.data, _dtype_code(X), labels.ctypes.data, B, N, K, d,
                               C_prev.ctypes.data, C_out.ctypes.data, sums.ctypes.data, counts.ctypes.data,
                               nthreads or threads())
    if rc:
        raise ValueError(f"oracle_update failed ({rc})")
    return C_out, sums, counts


def cost(X: np.ndarray, C: np.ndarray, labels: np.ndarray) -> np.ndarray:
    """Per-batch objective sum_i ||x_i - C[a_i]||^2 (C taken as given, in float64)."""
    X = _c(X)
    B, N, d = X.shape
    K = C.shape[1]
    C64 = _c(C, np.float64)
    labels = _c(labels, np.int32)
    J = np.empty(B, dtype=np.float64)
    rc = _load().oracle_cost(X.ctypes.data, _dtype_code(X), C64.ctypes.data, labels.ctypes.data, B, N, K, d,
                             J.ctypes.data)
    if rc:
        raise ValueError(f"oracle_cost failed ({rc})")
    return J


def lloyd(X: np.ndarray, C_init: np.ndarray, iters: int, nthreads: int | None = None):
    """`iters` Lloyd iterations: (labels of the last assignment, final C, objective [iters, B])."""
    X = _c(X)
    B, N, d = X.shape
    K = C_init.shape[1]
    C_init = _c(C_init, np.float32)
    labels = np.empty((B, N), dtype=np.int32)
    C_out = np.empty_like(C_init)
    obj = np.empty((iters, B), dtype=np.float64)
    rc = _load().oracle_lloyd(X.ctypes.data, _dtype_code(X), C_init.ctypes.data, B, N, K, d, iters,
                              labels.ctypes.data, C_out.ctypes.data, obj.ctypes.data, nthreads or threads())
    if rc:
        raise ValueError(f"oracle_lloyd failed ({rc})")
    return labels, C_out, obj


def lloyd_tol(X: np.ndarray, C_init: np.ndarray, max_iters: int, tol: float, nthreads: int | None = None):
    """Lloyd iterations until every batch's squared centroid shift is <= tol (or max_iters).

    Returns (iters_run, labels of the last assignment, final C, objective [iters_run, B],
    shift [iters_run, B]).
    """
    X = _c(X)
    B, N, d = X.shape
    K = C_init.shape[1]
    C_init = _c(C_init, np.float32)
    labels = np.empty((B, N), dtype=np.int32)
    C_out = np.empty_like(C_init)
    obj = np.empty((max_iters, B), dtype=np.float64)
    shift = np.empty((max_iters, B), dtype=np.float64)
    run = np.zeros(1, dtype=np.int32)
    rc = _load().oracle_lloyd_tol(X.ctypes.data, _dtype_code(X), C_init.ctypes.data, B, N, K, d, max_iters,
                                  float(tol), labels.ctypes.data, C_out.ctypes.data, obj.ctypes.data,
                                  run.ctypes.data, shift.ctypes.data, nthreads or threads())
    if rc:
        raise ValueError(f"oracle_lloyd_tol failed ({rc})")
    t = int(run[0])
    return t, labels, C_out, obj[:t], shift[:t]
