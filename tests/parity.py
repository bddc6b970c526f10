"""Comparison rules between the CUDA path and the CPU oracle.

Tolerances (the stated bar for this method):
  * labels: identical wherever the oracle's relative top-2 gap (d2 - d1) / d2 is
    at least TAU_LABEL (1e-3 for fp16 inputs, 1e-5 for fp32); below it, the GPU
    label must be a near-minimiser, dist(gpu label) <= d1 + tau * d2.  The
    number of such near ties is returned for reporting.
  * mindist: |m_gpu - m_oracle(gpu label)| <= tau_m(d) * (||x||^2 + ||c||^2) + 1e-6,
    the fp32 rounding scale of the expansion ||x||^2 + ||c||^2 - 2 x.c, with
    tau_m(d) = max(1e-5, d * 2^-24): x.c and ||x||^2 are fp32 sums of d terms, whose
    first-order error bound is gamma_d ~ d * u (u = 2^-24) times the sum of the
    terms' magnitudes, itself at most (||x||^2 + ||c||^2) / 2 for x.c.
  * sort, counts, offsets: bit-exact.
  * centroids: ||c_gpu - c_ref||_inf <= 1e-4 * max(||c_ref||_inf, 1e-6) per
    centroid; empty clusters bit-identical to the previous centroid.
"""
from __future__ import annotations

import numpy as np

import oracle

TAU_LABEL = {"f16": 1e-3, "f32": 1e-5}
TAU_MIND = 1e-5


def tau_mind(d: int) -> float:
    return max(TAU_MIND, d * 2.0 ** -24)
TAU_CENTROID = 1e-4


def dtype_name(X: np.ndarray) -> str:
    return "f16" if X.dtype == np.float16 else "f32"


def check_labels(X, C, gpu_labels, gpu_mindist=None, rows=None):
    """Check GPU labels (and mindist) for the flattened rows (all if None). Returns the near-tie count."""
    tau = TAU_LABEL[dtype_name(X)]
    B, N, d = X.shape
    code = oracle.F16 if X.dtype == np.float16 else oracle.F32
    chat = oracle.round_centroids(C, code)
    ref, d1, d2 = oracle.assign(X, C, rows=rows, chat=chat)
    ref, d1, d2 = ref.reshape(-1), d1.reshape(-1), d2.reshape(-1)
    flat = np.arange(B * N) if rows is None else np.asarray(rows)
    gl = np.asarray(gpu_labels).reshape(-1)[flat]
    assert gl.min() >= 0 and gl.max() < C.shape[1], "GPU label out of range"
    gap = (d2 - d1) / np.maximum(d2, np.finfo(np.float64).tiny)
    clear = gap >= tau
    bad = np.nonzero(clear & (gl != ref))[0]
    assert bad.size == 0, (f"{bad.size} labels differ at clear points; first rows {flat[bad[:5]]}, "
                           f"gpu {gl[bad[:5]]} oracle {ref[bad[:5]]} gap {gap[bad[:5]]}")
    Xf = X.reshape(B * N, d)
    bidx = flat // N
    xs = Xf[flat].astype(np.float64)
    cg = chat[bidx, gl]
    dist_g = ((xs - cg) ** 2).sum(axis=1)
    near = ~clear
    if near.any():
        ok = dist_g[near] <= d1[near] + tau * d2[near]
        assert ok.all(), f"{(~ok).sum()} near-tie labels are not near-minimisers"
    if gpu_mindist is not None:
        gm = np.asarray(gpu_mindist).reshape(-1)[flat].astype(np.float64)
        scale = (xs ** 2).sum(axis=1) + (cg ** 2).sum(axis=1)
        err = np.abs(gm - dist_g)
        lim = tau_mind(d) * scale + 1e-6
        worst = np.argmax(err / lim)
        assert (err <= lim).all(), (f"mindist off: row {flat[worst]} gpu {gm[worst]} ref {dist_g[worst]} "
                                    f"err {err[worst]} lim {lim[worst]}")
    return int(near.sum())


def check_sort(labels, K, gpu_sidx, gpu_counts, gpu_offsets=None):
    sidx, counts, offsets = oracle.sort_labels(np.asarray(labels), K)
    assert np.array_equal(np.asarray(gpu_counts), counts), "counts differ"
    assert np.array_equal(np.asarray(gpu_sidx), sidx), "sorted_idx differs"
    if gpu_offsets is not None:
        assert np.array_equal(np.asarray(gpu_offsets), offsets), "offsets differ"


def check_centroids(X, labels, C_prev, gpu_C, gpu_counts=None, gpu_sums=None):
    C_ref, sums_ref, counts_ref = oracle.update(X, np.asarray(labels), C_prev)
    gpu_C = np.asarray(gpu_C)
    if gpu_counts is not None:
        assert np.array_equal(np.asarray(gpu_counts), counts_ref), "counts differ"
    empty = counts_ref == 0
    assert np.array_equal(gpu_C[empty].view(np.uint32), np.asarray(C_prev)[empty].view(np.uint32)), \
        "an empty cluster did not keep its centroid"
    ref_inf = np.abs(C_ref.astype(np.float64)).max(axis=-1)
    err = np.abs(gpu_C.astype(np.float64) - C_ref.astype(np.float64)).max(axis=-1)
    lim = TAU_CENTROID * np.maximum(ref_inf, 1e-6)
    bad = np.nonzero(err > lim)
    assert bad[0].size == 0, f"{bad[0].size} centroids off; worst rel {(err / np.maximum(ref_inf, 1e-6)).max():.3e}"
    if gpu_sums is not None:
        n = np.maximum(counts_ref, 1)[..., None]
        # sums compared as means, on the same relative scale as the centroids
        serr = np.abs(np.asarray(gpu_sums, dtype=np.float64) - sums_ref).max(axis=-1) / n[..., 0]
        assert (serr <= lim + 1e-6).all(), "sums off"
    return C_ref
