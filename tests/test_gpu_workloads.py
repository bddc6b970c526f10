"""Parity at the full workload sizes, in the launch configuration the benchmark uses.

Lock-step protocol: at each iteration the oracle takes the GPU's centroids C_t; the GPU's labels are
checked on 65,536 sampled rows (the oracle's assignment is O(K d) per row; every row at one iteration of
the metric's workload), the argsort and counts bit-exactly over all points, and the update over all
points, for every iteration of each workload.  A multi-iteration call is checked at its end.
"""
import numpy as np
import pytest

import synth
from parity import check_centroids, check_labels, check_sort

torch = pytest.importorskip("torch")
import flashassign_b200 as km  # noqa: E402

pytestmark = pytest.mark.gpu


def cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def sample_rows(B, N, n, seed):
    rng = np.random.default_rng(seed)
    rows = rng.choice(B * N, size=min(n, B * N), replace=False)
    # always include the first and last rows of every batch (tile edges)
    edges = np.concatenate([np.arange(B) * N, np.arange(B) * N + N - 1])
    return np.unique(np.concatenate([rows, edges]))


def lockstep(w, iters, nsample, full_at=None):
    """Every iteration of the workload in lock step with the oracle; at iteration `full_at` every
    label is checked."""
    X = synth.points(w)
    C = synth.init_centroids(w, X)
    Xg = cuda(X)
    near = checked = 0
    km.assign_rescans()
    for t in range(iters):
        lab, C_next, obj = km.lloyd(Xg, cuda(C), 1)
        torch.cuda.synchronize()
        lab, C_next = lab.cpu().numpy(), C_next.cpu().numpy()
        rows = None if t == full_at else sample_rows(w.B, w.N, nsample, seed=t)
        near += check_labels(X, C, lab, rows=rows)
        checked += w.B * w.N if rows is None else len(rows)
        sidx, counts, offs = km.sort_labels(cuda(lab), w.K)
        check_sort(lab, w.K, sidx.cpu().numpy(), counts.cpu().numpy(), offs.cpu().numpy())
        check_centroids(X, lab, C, C_next)
        C = C_next
    assert km.device_fault() == 0
    print(f"{w.name}: {iters} iterations in lock step, {checked} labels checked, {near} near-tie points "
          f"(relative top-2 gap below the label tolerance), {km.assign_rescans()} points re-scanned exactly")
    return X, C, near


def test_workload1_small_fp32_full_lockstep():
    w = synth.WORKLOADS[1]
    lockstep(w, w.iters, nsample=w.B * w.N)


def test_workload2_metric_configuration():
    # all 20 iterations; 65,536 labels per iteration and, at the last one, all 2,097,152
    w = synth.WORKLOADS[2]
    X, C, near = lockstep(w, w.iters, nsample=65536, full_at=w.iters - 1)
    # and a multi-iteration call, as the benchmark makes it: check its last assignment
    Xg = cuda(X)
    lab_a, C_a, _ = km.lloyd(Xg, cuda(C), 4)        # four more iterations ...
    lab_b, C_b, _ = km.lloyd(Xg, cuda(C), 3)        # ... whose first three give the last one's input
    torch.cuda.synchronize()
    C3 = C_b.cpu().numpy()
    check_labels(X, C3, lab_a.cpu().numpy(), rows=sample_rows(w.B, w.N, 65536, seed=99))


def test_workload3_zipf_hot_clusters():
    w = synth.WORKLOADS[3]
    lockstep(w, w.iters, nsample=65536)


def test_workload4_large_k():
    w = synth.WORKLOADS[4]
    lockstep(w, w.iters, nsample=65536)


def test_wide_points_d512_k65536():
    # the d = 512 shape of the page's end-to-end table, on the chunked tensor-core path
    w = synth.WORKLOADS[6]
    lockstep(w, 1, nsample=4096)


def test_very_wide_points_d4096_split_d():
    # d = 4096 on the split-D tensor-core path (points and centroids both streamed along d)
    w = synth.WORKLOADS[7]
    lockstep(w, w.iters, nsample=4096)


def test_workload5_host_resident_fp32_chunked():
    """2^27 x 128 fp32 points (64 GiB) in pinned host memory, streamed in 2^23-row chunks."""
    import time
    import oracle
    w = synth.WORKLOADS[5]
    Xh = torch.empty((w.B, w.N, w.d), dtype=torch.float32).pin_memory()
    X = Xh.numpy()
    synth.points(w, out=X)
    C = synth.init_centroids(w, X)
    lab_h = torch.empty((w.B, w.N), dtype=torch.int32).pin_memory()
    km.lib().km_set_chunk_rows(w.chunk_rows)
    km.assign_rescans()
    try:
        for t in range(w.iters):
            t0 = time.perf_counter()
            lab_h, C_next, obj = km.lloyd(Xh, torch.from_numpy(C).cuda(), 1, labels=lab_h)
            torch.cuda.synchronize()
            print(f"workload 5 iteration {t}: {time.perf_counter() - t0:.2f} s")
            lab = lab_h.numpy()
            C_next = C_next.cpu().numpy()
            near = check_labels(X, C, lab, rows=sample_rows(w.B, w.N, 65536, seed=50 + t))
            print(f"workload 5 iteration {t}: {near} near-tie points of 65536 checked rows, "
                  f"{km.assign_rescans()} points re-scanned exactly")
            # argsort and counts over every point
            sidx, counts, offs = km.sort_labels(torch.from_numpy(lab).cuda(), w.K)
            check_sort(lab, w.K, sidx.cpu().numpy(), counts.cpu().numpy(), offs.cpu().numpy())
            # update: the oracle's means of a sample of clusters, from their member rows
            rng = np.random.default_rng(60 + t)
            ks = np.sort(rng.choice(w.K, 256, replace=False))
            members = np.isin(lab[0], ks)
            Xs = np.ascontiguousarray(X[0][members])[None]
            remap = np.full(w.K, -1, dtype=np.int32)
            remap[ks] = np.arange(len(ks), dtype=np.int32)
            C_sub, _, _ = oracle.update(Xs, remap[lab[0][members]][None], C[:, ks])
            err = np.abs(C_next[0, ks].astype(np.float64) - C_sub[0]).max(axis=1)
            lim = 1e-4 * np.maximum(np.abs(C_sub[0]).max(axis=1), 1e-6)
            assert (err <= lim).all(), (err / lim).max()
            C = C_next
    finally:
        km.lib().km_set_chunk_rows(0)
    assert km.device_fault() == 0
