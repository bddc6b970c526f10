"""Python binding of libkm.so, the B200 batched exact Lloyd k-means library.

Argument marshalling only: every step runs in the CUDA library behind the C ABI
of include/km.h.  PyTorch supplies device memory and the current CUDA stream.
There is no fallback: if libkm.so is missing or a call fails, an exception is
raised.  Build the library with ``python -m flashassign_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkm.so")

KM_F32, KM_F16 = 0, 1
STATUS = {0: "KM_OK", 1: "KM_E_INVALID", 2: "KM_E_UNSUPPORTED", 3: "KM_E_NOMEM", 4: "KM_E_CUDA", 5: "KM_E_TIMEOUT"}

# name -> (restype, argtypes), mirroring include/km.h
_P, _I64, _INT = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
SIGNATURES = {
    "km_assign": (_INT, [_P, _P, _I64, _I64, _I64, _I64, _INT, _P, _P, _P]),
    "km_assign_objective": (_INT, [_P, _P, _I64, _I64, _I64, _I64, _INT, _P, _P, _P, _P]),
    "km_sort_labels": (_INT, [_P, _I64, _I64, _I64, _P, _P, _P, _P]),
    "km_update": (_INT, [_P, _P, _I64, _I64, _I64, _I64, _INT, _P, _P, _P, _P]),
    "km_lloyd": (_INT, [_P, _P, _I64, _I64, _I64, _I64, _INT, _INT, _P, _P, _P, _P]),
    "km_lloyd_tol": (_INT, [_P, _P, _I64, _I64, _I64, _I64, _INT, _INT, ctypes.c_double, _P, _P, _P, _P, _P]),
    "km_set_chunk_rows": (None, [_I64]),
    "km_release_cached": (_INT, []),
    "km_status_string": (ctypes.c_char_p, [_INT]),
    "km_last_error": (ctypes.c_char_p, []),
    "km_device_fault": (_INT, [ctypes.POINTER(ctypes.c_int32), _P]),
    "km_assign_rescans": (_INT, [ctypes.POINTER(ctypes.c_int64), _P]),
    "km_assign_noalloc": (_INT, [_P, _P, _I64, _I64, _I64, _I64, _INT, _P, _P, _P]),
    "km_assign_dense": (_INT, [_P, _P, _I64, _I64, _I64, _I64, _INT, _P, _P, _P]),
    "km_update_sums": (_INT, [_P, _P, _I64, _I64, _I64, _I64, _INT, _P, _P, _P]),
    "km_finalize": (_INT, [_P, _P, _I64, _I64, _I64, _P, _P]),
    "km_update_scatter": (_INT, [_P, _P, _I64, _I64, _I64, _I64, _INT, _P, _P, _P, _P]),
    "km_assign_noalloc_limit": (ctypes.c_size_t, []),
    "km_trace_enable": (None, [_INT]),
    "km_trace_read": (_INT, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64), _INT]),
}
PHASES = ("prep", "assign", "sort", "update", "finalize", "other")


class KMError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)}: {detail}")
        self.status = status
        self.detail = detail


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libkm.so with argument types set (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} not found: build it with `python -m flashassign_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def check(fn: str, status: int) -> None:
    if status != 0:
        raise KMError(fn, status, lib().km_last_error().decode())


# ---- torch-level helpers (marshalling only) -------------------------------------

def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(X) -> int:
    torch = _torch()
    if X.dtype == torch.float16:
        return KM_F16
    if X.dtype == torch.float32:
        return KM_F32
    raise TypeError(f"X must be float16 or float32, got {X.dtype}")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _require(t, shape, dtype, name):
    torch = _torch()
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)}")
    return t


def assign(X, C, labels=None, mindist=None, stream=None):
    """FlashAssign: (labels [B,N] int32, mindist [B,N] fp32) for X [B,N,d], C [B,K,d] fp32."""
    torch = _torch()
    B, N, d = X.shape
    K = C.shape[1]
    _require(C, (B, K, d), torch.float32, "C")
    if labels is None:
        labels = torch.empty((B, N), dtype=torch.int32, device=X.device)
    if mindist is None:
        mindist = torch.empty((B, N), dtype=torch.float32, device=X.device)
    check("km_assign", lib().km_assign(_ptr(X), _ptr(C), B, N, K, d, _dtype_code(X), _ptr(labels), _ptr(mindist),
                                       _stream(stream)))
    return labels, mindist


def assign_objective(X, C, labels=None, mindist=None, stream=None):
    """assign() plus the per-problem objective sum_i mindist (fp64 [B]) from the assignment kernels."""
    torch = _torch()
    B, N, d = X.shape
    K = C.shape[1]
    _require(C, (B, K, d), torch.float32, "C")
    if labels is None:
        labels = torch.empty((B, N), dtype=torch.int32, device=X.device)
    if mindist is None:
        mindist = torch.empty((B, N), dtype=torch.float32, device=X.device)
    objective = torch.empty(B, dtype=torch.float64, device=X.device)
    check("km_assign_objective", lib().km_assign_objective(_ptr(X), _ptr(C), B, N, K, d, _dtype_code(X),
                                                           _ptr(labels), _ptr(mindist), _ptr(objective),
                                                           _stream(stream)))
    return labels, mindist, objective


def assign_dense(X, C, labels=None, mindist=None, stream=None):
    """Baseline: the assignment with the N x K score matrix materialised in HBM (same results as assign)."""
    torch = _torch()
    B, N, d = X.shape
    K = C.shape[1]
    _require(C, (B, K, d), torch.float32, "C")
    if labels is None:
        labels = torch.empty((B, N), dtype=torch.int32, device=X.device)
    if mindist is None:
        mindist = torch.empty((B, N), dtype=torch.float32, device=X.device)
    check("km_assign_dense", lib().km_assign_dense(_ptr(X), _ptr(C), B, N, K, d, _dtype_code(X), _ptr(labels),
                                                   _ptr(mindist), _stream(stream)))
    return labels, mindist


def update_scatter(X, labels, C_prev, stream=None):
    """Baseline: the update with one atomic per point coordinate (same results as update)."""
    torch = _torch()
    B, N, d = X.shape
    K = C_prev.shape[1]
    _require(labels, (B, N), torch.int32, "labels")
    _require(C_prev, (B, K, d), torch.float32, "C_prev")
    C_out = C_prev.clone()
    sums = torch.empty((B, K, d), dtype=torch.float32, device=X.device)
    counts = torch.empty((B, K), dtype=torch.int32, device=X.device)
    check("km_update_scatter", lib().km_update_scatter(_ptr(X), _ptr(labels), B, N, K, d, _dtype_code(X),
                                                       _ptr(sums), _ptr(counts), _ptr(C_out), _stream(stream)))
    return C_out, sums, counts


def sort_labels(labels, K: int, stream=None):
    """Stable argsort of labels [B,N]: (sorted_idx [B,N], counts [B,K], offsets [B,K+1])."""
    torch = _torch()
    B, N = labels.shape
    _require(labels, (B, N), torch.int32, "labels")
    sidx = torch.empty((B, N), dtype=torch.int32, device=labels.device)
    counts = torch.empty((B, K), dtype=torch.int32, device=labels.device)
    offsets = torch.empty((B, K + 1), dtype=torch.int32, device=labels.device)
    check("km_sort_labels", lib().km_sort_labels(_ptr(labels), B, N, K, _ptr(sidx), _ptr(counts), _ptr(offsets),
                                                 _stream(stream)))
    return sidx, counts, offsets


def update(X, labels, C_prev, stream=None):
    """Sort-Inverse Update: (C_out [B,K,d] fp32, sums [B,K,d] fp32, counts [B,K] int32)."""
    torch = _torch()
    B, N, d = X.shape
    K = C_prev.shape[1]
    _require(labels, (B, N), torch.int32, "labels")
    _require(C_prev, (B, K, d), torch.float32, "C_prev")
    C_out = C_prev.clone()
    sums = torch.empty((B, K, d), dtype=torch.float32, device=X.device)
    counts = torch.empty((B, K), dtype=torch.int32, device=X.device)
    check("km_update", lib().km_update(_ptr(X), _ptr(labels), B, N, K, d, _dtype_code(X), _ptr(sums), _ptr(counts),
                                       _ptr(C_out), _stream(stream)))
    return C_out, sums, counts


def update_sums(X, labels, K: int, stream=None):
    """The first half of the update: (sums [B,K,d] fp32, counts [B,K] int32); no centroid is written."""
    torch = _torch()
    B, N, d = X.shape
    _require(labels, (B, N), torch.int32, "labels")
    sums = torch.empty((B, K, d), dtype=torch.float32, device=X.device)
    counts = torch.empty((B, K), dtype=torch.int32, device=X.device)
    check("km_update_sums", lib().km_update_sums(_ptr(X), _ptr(labels), B, N, K, d, _dtype_code(X), _ptr(sums),
                                                 _ptr(counts), _stream(stream)))
    return sums, counts


def finalize(sums, counts, C_prev, stream=None):
    """The second half: sums / counts where counts > 0, else the previous centroid."""
    torch = _torch()
    B, K, d = C_prev.shape
    _require(sums, (B, K, d), torch.float32, "sums")
    _require(counts, (B, K), torch.int32, "counts")
    C_out = C_prev.clone()
    check("km_finalize", lib().km_finalize(_ptr(sums), _ptr(counts), B, K, d, _ptr(C_out), _stream(stream)))
    return C_out


def lloyd(X, C_init, iters: int, labels=None, C_out=None, objective=None, stream=None):
    """`iters` Lloyd iterations: (labels of the last assignment, final centroids, objective [iters,B])."""
    torch = _torch()
    B, N, d = X.shape
    K = C_init.shape[1]
    _require(C_init, (B, K, d), torch.float32, "C_init")
    dev = C_init.device
    if labels is None:
        labels = torch.empty((B, N), dtype=torch.int32, device=dev if X.is_cuda else "cpu",
                             pin_memory=not X.is_cuda)
    if C_out is None:
        C_out = torch.empty_like(C_init)
    if objective is None and iters > 0:
        objective = torch.empty((iters, B), dtype=torch.float32, device=dev)
    check("km_lloyd", lib().km_lloyd(_ptr(X), _ptr(C_init), B, N, K, d, _dtype_code(X), iters, _ptr(labels),
                                     _ptr(C_out), _ptr(objective), _stream(stream)))
    return labels, C_out, objective


def lloyd_tol(X, C_init, max_iters: int, tol: float, labels=None, C_out=None, objective=None, stream=None):
    """Lloyd iterations until every batch's squared centroid shift is <= tol (or max_iters):
    (labels, centroids, objective [max_iters, B] -- rows past the stop unwritten, iterations run)."""
    torch = _torch()
    B, N, d = X.shape
    K = C_init.shape[1]
    _require(C_init, (B, K, d), torch.float32, "C_init")
    dev = C_init.device
    if labels is None:
        labels = torch.empty((B, N), dtype=torch.int32, device=dev)
    if C_out is None:
        C_out = torch.empty_like(C_init)
    if objective is None:
        objective = torch.full((max_iters, B), float("nan"), dtype=torch.float32, device=dev)
    iters_run = torch.zeros(1, dtype=torch.int32, device=dev)
    check("km_lloyd_tol", lib().km_lloyd_tol(_ptr(X), _ptr(C_init), B, N, K, d, _dtype_code(X), max_iters, float(tol),
                                             _ptr(labels), _ptr(C_out), _ptr(objective), _ptr(iters_run),
                                             _stream(stream)))
    return labels, C_out, objective, iters_run


def device_fault(stream=None) -> int:
    """Read and clear the device fault word (0 = no bounded wait expired)."""
    code = ctypes.c_int32(0)
    check("km_device_fault", lib().km_device_fault(ctypes.byref(code), _stream(stream)))
    return int(code.value)


def assign_rescans(stream=None) -> int:
    """Read and clear the count of points handed to the exact re-scan (see include/km.h)."""
    n = ctypes.c_int64(0)
    check("km_assign_rescans", lib().km_assign_rescans(ctypes.byref(n), _stream(stream)))
    return int(n.value)


def trace_enable(on: bool = True) -> None:
    lib().km_trace_enable(1 if on else 0)


def trace_read() -> dict:
    """Per-phase GPU milliseconds and kernel launch counts recorded since the last read."""
    n = len(PHASES)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    check("km_trace_read", lib().km_trace_read(ms, cnt, n))
    return {p: (float(ms[i]), int(cnt[i])) for i, p in enumerate(PHASES)}
