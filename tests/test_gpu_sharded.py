"""The N-sharded iteration on the GPU path: the library's steps and an NCCL all-reduce.

One GPU is available, so the process group has one rank (the all-reduce runs, and adds nothing);
the exchange between several ranks is covered on CPU ranks by test_sharded.py.  The sharded loop
must then equal km_lloyd on the same points.
"""
import datetime
import socket

import numpy as np
import pytest

import synth
from parity import check_centroids, check_labels

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402

import flashassign_b200 as km  # noqa: E402
from flashassign_b200.sharded import lloyd_sharded  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("dt,d,K", [("f16", 128, 300), ("f32", 128, 100), ("f32", 16, 10), ("f16", 1024, 600)])
def test_one_rank_sharded_loop_equals_lloyd(nccl_group, dt, d, K):
    w = synth.small(B=2, N=3000, d=d, K=K, dtype=dt, ncomp=K, sigma=0.3, seed=6000 + d + K)
    X = synth.points(w)
    C0 = synth.init_centroids(w, X)
    Xg, Cg = torch.from_numpy(X).cuda(), torch.from_numpy(C0).cuda()
    lab_s, C_s, obj_s = lloyd_sharded(Xg, Cg, 3)
    lab_l, C_l, obj_l = km.lloyd(Xg, Cg, 3)
    torch.cuda.synchronize()
    assert (lab_s == lab_l).float().mean().item() > 0.9999
    torch.testing.assert_close(C_s, C_l, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(obj_s.float(), obj_l, rtol=1e-5, atol=0)
    # and one more step of the sharded halves against the oracle
    sums, counts = km.update_sums(Xg, lab_s, K)
    C_next = km.finalize(sums, counts, C_s)
    torch.cuda.synchronize()
    check_centroids(X, lab_s.cpu().numpy(), C_s.cpu().numpy(), C_next.cpu().numpy(), counts.cpu().numpy())
    assert km.device_fault() == 0
