"""The N-sharded iteration (flashassign_b200.sharded): the exchange logic on two CPU ranks (gloo).

Each rank holds every other point of each problem; the per-rank steps are the oracle's (assign,
sums and counts of a labelling, division), so the test checks what the sharding adds -- the
all-reduce of sums, counts and objective between the two halves of the update -- against one
process running the oracle over all the points.
"""
import os
import socket

import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

from flashassign_b200.sharded import Ops, lloyd_sharded  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_ops() -> Ops:
    def assign(X, C):
        B, N, _ = X.shape
        lab, d1, _ = oracle.assign(X.numpy(), C.numpy())
        return torch.from_numpy(lab.reshape(B, N)), torch.from_numpy(d1.reshape(B, N).sum(axis=1))

    def update_sums(X, labels, K):
        B, _, d = X.shape
        _, sums, counts = oracle.update(X.numpy(), labels.numpy(), np.zeros((B, K, d), np.float32))
        return torch.from_numpy(sums), torch.from_numpy(counts)

    def finalize(sums, counts, C_prev):
        s, n = sums.numpy(), counts.numpy()
        C = C_prev.numpy().copy()
        nz = n > 0
        C[nz] = (s[nz] / n[nz][:, None]).astype(np.float32)
        return torch.from_numpy(C)

    return Ops(assign=assign, update_sums=update_sums, finalize=finalize)


def _worker(rank, world, port, X, C0, iters, out_dir):
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        shard = torch.from_numpy(np.ascontiguousarray(X[:, rank::world]))
        labels, C, obj = lloyd_sharded(shard, torch.from_numpy(C0), iters, ops=_oracle_ops())
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), labels=labels.numpy(), C=C.numpy(), obj=obj.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dt,d,K", [("f32", 16, 12), ("f16", 64, 30)])
def test_two_rank_shards_equal_one_process_over_all_points(tmp_path, dt, d, K):
    w = synth.small(B=2, N=1501, d=d, K=K, dtype=dt, ncomp=K, sigma=0.3, seed=5000 + d)
    X = synth.points(w)
    C0 = synth.init_centroids(w, X)
    iters, world = 4, 2
    mp.spawn(_worker, args=(world, _free_port(), X, C0, iters, str(tmp_path)), nprocs=world, join=True)
    ref_labels, ref_C, ref_obj = oracle.lloyd(X, C0, iters)
    Cs = []
    for r in range(world):
        got = np.load(tmp_path / f"rank{r}.npz")
        # the last assignment of this rank's points equals the single-process one
        assert np.array_equal(got["labels"], ref_labels[:, r::world])
        Cs.append(got["C"])
        np.testing.assert_allclose(got["obj"], ref_obj, rtol=1e-9)
    # every rank holds the same centroids, those of one process over all the points (sums added in
    # another order: fp32 of the double means, within one unit in the last place)
    assert np.array_equal(Cs[0], Cs[1])
    np.testing.assert_allclose(Cs[0], ref_C, rtol=2e-7, atol=1e-7)
