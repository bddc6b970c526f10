"""Lloyd iterations with the points of every problem sharded across processes (one per GPU).

Every rank holds a shard X_r [B, N_r, d] of each of the B problems' points and the same centroids.
An iteration is the method's iteration (papernotes.org "Flash-KMeans" page, 整体框架) with one
exchange added between the two halves of the update: each rank assigns its own points and reduces
them into per-cluster sums and counts (the sort-inverse gather-reduce), one all-reduce adds the
sums (fp32 [B,K,d]) and counts (int32 [B,K]) over the ranks, and every rank finalises the same
centroids.  The assignment needs no exchange (each point only meets the centroids), so the only
traffic per iteration is 4*B*K*(d+1) bytes per rank, independent of N.

The step functions are those of the library (`flashassign_b200.assign_objective`, `update_sums`,
`finalize`) unless `ops` supplies others with the same signatures (the multi-process tests run the
exchange logic on CPU ranks that way); this module only moves their results between the ranks.
Every rank takes the same collective steps in the same order.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable


@dataclass(frozen=True)
class Ops:
    """The three per-rank steps: assign(X, C) -> (labels, objective [B] fp64 of this shard);
    update_sums(X, labels, K) -> (sums, counts); finalize(sums, counts, C_prev) -> C_new."""
    assign: Callable
    update_sums: Callable
    finalize: Callable


def library_ops() -> Ops:
    import flashassign_b200 as km

    def assign(X, C):
        labels, _, objective = km.assign_objective(X, C)
        return labels, objective

    return Ops(assign=assign, update_sums=km.update_sums, finalize=km.finalize)


def lloyd_sharded(X_local, C_init, iters: int, group=None, ops: Ops | None = None):
    """`iters` Lloyd iterations over the union of every rank's shard.

    Returns (labels of this rank's points from the last assignment, the final centroids, the
    objective per iteration and problem [iters, B] summed over all ranks' points)."""
    import torch
    import torch.distributed as dist

    ops = ops or library_ops()
    K = C_init.shape[1]
    C = C_init.clone()
    objective = []
    labels = None
    for _ in range(iters):
        labels, obj = ops.assign(X_local, C)
        sums, counts = ops.update_sums(X_local, labels, K)
        dist.all_reduce(sums, group=group)
        dist.all_reduce(counts, group=group)
        dist.all_reduce(obj, group=group)
        C = ops.finalize(sums, counts, C)
        objective.append(obj)
    return labels, C, torch.stack(objective) if objective else None
