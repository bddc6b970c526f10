"""Seeded synthetic inputs shared by the CPU oracle, the tests and the benchmark.

This module draws random numbers only: Gaussian-mixture points, the component
of each point, and the K distinct rows used as initial centroids.  It contains
none of the k-means arithmetic, so that the oracle and the CUDA path share no
code beyond the bytes they are fed.

The workloads mirror the benchmark shapes on the Flash-KMeans pages
(papernotes.org "Flash-KMeans: Fast and Memory-Efficient Exact K-Means",
section 实验关键数据: FP16, d=128, sweeps over N, K and the batch B; tilnote.io
page: an FP32, d=128 large-tensor benchmark held in pinned CPU memory and
streamed in chunks).  The pages measure on synthetic sweeps, not on a dataset.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile libsynth.so next to this file (plain C, pthreads)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-pthread", "-o", _SO, src, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.synth_philox4x32_10.argtypes = [ctypes.POINTER(ctypes.c_uint32)] * 3
        lib.synth_uniform53.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        lib.synth_mixture.restype = ctypes.c_int
        lib.synth_mixture.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                      ctypes.c_double, ctypes.c_double, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        _lib = lib
    return _lib


def philox4x32_10(ctr, key):
    """One Philox4x32-10 block (exposed for the known-answer test)."""
    lib = _load()
    c = (ctypes.c_uint32 * 4)(*[int(v) & 0xFFFFFFFF for v in ctr])
    k = (ctypes.c_uint32 * 2)(*[int(v) & 0xFFFFFFFF for v in key])
    o = (ctypes.c_uint32 * 4)()
    lib.synth_philox4x32_10(c, k, o)
    return [int(v) for v in o]


def uniform53(seed: int, batch: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _load().synth_uniform53(seed, batch, n, out.ctypes.data)
    return out


def normals(seed: int, stream: int, batch: int, row0: int, nrows: int, d: int) -> np.ndarray:
    out = np.empty((nrows, d), dtype=np.float64)
    _load().synth_normal(seed, stream, batch, row0, nrows, d, out.ctypes.data)
    return out


@dataclass(frozen=True)
class Workload:
    """A batched Lloyd problem: B independent problems of N points in d dims, K centroids."""
    name: str
    B: int
    N: int
    d: int
    K: int
    dtype: str              # "f16" or "f32": the dtype X is stored and multiplied in
    ncomp: int              # mixture components
    sigma: float            # per-coordinate std of each component
    iters: int
    center: str = "normal"  # "normal": N(0,1)^d centres; "uniform": U[lo, hi)^d centres
    c_lo: float = -10.0
    c_hi: float = 10.0
    zipf: float = 0.0       # 0: equal weights; s > 0: weight of rank r proportional to r^-s
    seed: int = 0x6B6D0000
    host: bool = False      # X held in pinned host memory and streamed in chunks
    chunk_rows: int = 0

    @property
    def np_dtype(self):
        return np.float16 if self.dtype == "f16" else np.float32

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "f16" else 4

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads: shapes and distributions from the benchmark descriptions above.
WORKLOADS = {
    1: Workload("b1_n4096_d16_k8_f32", 1, 4096, 16, 8, "f32", ncomp=8, sigma=1.0, iters=10,
                center="uniform", c_lo=-10.0, c_hi=10.0, seed=0x6B6D0001),
    2: Workload("b32_n65536_d128_k1024_f16", 32, 65536, 128, 1024, "f16", ncomp=1024, sigma=0.3,
                iters=20, seed=0x6B6D0002),
    3: Workload("b8_n262144_d128_k4096_f16_zipf1.2", 8, 262144, 128, 4096, "f16", ncomp=4096,
                sigma=0.2, iters=10, zipf=1.2, seed=0x6B6D0003),
    4: Workload("b1_n1048576_d128_k65536_f16", 1, 1 << 20, 128, 65536, "f16", ncomp=65536,
                sigma=0.25, iters=5, seed=0x6B6D0004),
    5: Workload("b1_n134217728_d128_k4096_f32_host", 1, 1 << 27, 128, 4096, "f32", ncomp=4096,
                sigma=0.3, iters=3, seed=0x6B6D0005, host=True, chunk_rows=1 << 23),
    # wide points: the d = 512 shape of the papernotes.org page's end-to-end table (N = 1M, K = 65536)
    6: Workload("b1_n1048576_d512_k65536_f16", 1, 1 << 20, 512, 65536, "f16", ncomp=65536,
                sigma=0.25, iters=3, seed=0x6B6D0006),
    # very wide points: d = 4096, the dense multimodal width the papernotes.org page names as the limit
    # of on-chip tiles (局限与展望), served by the split-D path
    7: Workload("b1_n262144_d4096_k4096_f16", 1, 1 << 18, 4096, 4096, "f16", ncomp=4096,
                sigma=0.25, iters=3, seed=0x6B6D0007),
}


def small(B=2, N=1000, d=64, K=40, dtype="f16", ncomp=None, sigma=0.3, seed=12345, **kw) -> Workload:
    """A small workload of the same family, for tests."""
    return Workload(f"small_b{B}_n{N}_d{d}_k{K}_{dtype}", B, N, d, K, dtype,
                    ncomp=ncomp if ncomp is not None else K, sigma=sigma, iters=kw.pop("iters", 3),
                    seed=seed, **kw)


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def points(w: Workload, row0: int = 0, nrows: int | None = None, out: np.ndarray | None = None,
           with_components: bool = False):
    """Rows [row0, row0+nrows) of every batch: array [B, nrows, d] in w's dtype."""
    if nrows is None:
        nrows = w.N - row0
    if out is None:
        out = np.empty((w.B, nrows, w.d), dtype=w.np_dtype)
    assert out.shape == (w.B, nrows, w.d) and out.dtype == w.np_dtype and out.flags.c_contiguous
    comp = np.empty((w.B, nrows), dtype=np.int32) if with_components else None
    rc = _load().synth_mixture(w.seed, w.B, w.N, w.d, w.ncomp, 0 if w.center == "normal" else 1,
                               w.c_lo, w.c_hi, w.sigma, w.zipf, row0, nrows,
                               1 if w.dtype == "f16" else 0, out.ctypes.data,
                               comp.ctypes.data if comp is not None else None, _threads())
    if rc != 0:
        raise MemoryError("synth_mixture: host allocation failed")
    return (out, comp) if with_components else out


def init_indices(w: Workload) -> np.ndarray:
    """K distinct row indices per batch (partial Fisher-Yates driven by Philox uniforms)."""
    if w.K > w.N:
        raise ValueError("K distinct initial points need K <= N")
    idx = np.empty((w.B, w.K), dtype=np.int64)
    for b in range(w.B):
        u = uniform53(w.seed ^ 0x5EED, b, w.K)
        swapped: dict[int, int] = {}
        for i in range(w.K):
            j = i + int(u[i] * (w.N - i))
            vi, vj = swapped.get(i, i), swapped.get(j, j)
            swapped[i], swapped[j] = vj, vi
            idx[b, i] = vj
    return idx


def init_centroids(w: Workload, X: np.ndarray) -> np.ndarray:
    """Initial centroids [B, K, d] fp32: the rows of X [B, N, d] picked by init_indices."""
    idx = init_indices(w)
    C = np.empty((w.B, w.K, w.d), dtype=np.float32)
    for b in range(w.B):
        C[b] = X[b, idx[b]].astype(np.float32)
    return C
