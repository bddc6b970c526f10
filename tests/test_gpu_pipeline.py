"""km_lloyd with X in pinned host memory: the chunked copy/compute pipeline.

The same iteration as the device path, with X streamed through two device
slots of R rows: results are checked against the device path on the same
inputs (1 chunk, 2 chunks, an odd number of chunks with a ragged tail) and,
over several iterations, against the oracle in lock step.
"""
import numpy as np
import pytest

import synth
from parity import check_centroids, check_labels

torch = pytest.importorskip("torch")
import flashassign_b200 as km  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def restore_chunk_rows():
    yield
    km.lib().km_set_chunk_rows(0)


def pinned(a):
    return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()


@pytest.mark.parametrize("dtype,d", [("f16", 128), ("f32", 16), ("f32", 128), ("f16", 320), ("f16", 1024)])
@pytest.mark.parametrize("chunk_rows", [0, 1500, 1000, 777])  # 0: default (one chunk per batch here)
def test_host_pipeline_matches_device_path(dtype, d, chunk_rows):
    w = synth.small(B=2, N=3000, d=d, K=70, dtype=dtype, ncomp=70, seed=31 + d)
    X = synth.points(w)
    C0 = torch.from_numpy(synth.init_centroids(w, X)).cuda()
    lab_d, C_d, obj_d = km.lloyd(torch.from_numpy(X).cuda(), C0, 1)
    km.lib().km_set_chunk_rows(chunk_rows)
    Xh = pinned(X)
    lab_h = torch.empty((w.B, w.N), dtype=torch.int32).pin_memory()
    lab_h, C_h, obj_h = km.lloyd(Xh, C0, 1, labels=lab_h)
    torch.cuda.synchronize()
    # same centroids in, same kernels: identical labels; sums accumulate per chunk, so the
    # centroids agree to fp32 rounding
    assert torch.equal(lab_h, lab_d.cpu())
    torch.testing.assert_close(C_h, C_d, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(obj_h, obj_d, rtol=1e-5, atol=0)
    assert km.device_fault() == 0


@pytest.mark.parametrize("dtype,d", [("f16", 128), ("f32", 32)])
def test_host_pipeline_lockstep_with_oracle(dtype, d):
    w = synth.small(B=2, N=5000, d=d, K=100, dtype=dtype, ncomp=100, seed=41)
    X = synth.points(w)
    C = synth.init_centroids(w, X)
    km.lib().km_set_chunk_rows(1234)  # 5 chunks per batch, ragged tail
    Xh = pinned(X)
    lab_h = torch.empty((w.B, w.N), dtype=torch.int32).pin_memory()
    for t in range(4):
        lab_h, C_next, _ = km.lloyd(Xh, torch.from_numpy(C).cuda(), 1, labels=lab_h)
        torch.cuda.synchronize()
        lab = lab_h.numpy().copy()
        check_labels(X, C, lab)
        C_next = C_next.cpu().numpy()
        check_centroids(X, lab, C, C_next)
        C = C_next


def test_host_pipeline_many_iterations_and_device_labels():
    w = synth.small(B=1, N=6000, d=128, K=50, dtype="f16", seed=43)
    X = synth.points(w)
    C0 = torch.from_numpy(synth.init_centroids(w, X)).cuda()
    km.lib().km_set_chunk_rows(2500)
    lab_dev = torch.empty((w.B, w.N), dtype=torch.int32, device="cuda")
    lab, C5, obj = km.lloyd(pinned(X), C0, 5, labels=lab_dev)
    lab_ref, C_ref, obj_ref = km.lloyd(torch.from_numpy(X).cuda(), C0, 5)
    torch.cuda.synchronize()
    assert (lab.cpu() == lab_ref.cpu()).float().mean() > 0.999
    torch.testing.assert_close(C5, C_ref, rtol=1e-4, atol=1e-5)
    torch.testing.assert_close(obj, obj_ref, rtol=1e-4, atol=0)


def test_pageable_host_memory_is_rejected():
    X = torch.zeros((1, 256, 64), dtype=torch.float16)  # not pinned
    C = torch.zeros((1, 4, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(km.KMError) as e:
        km.lloyd(X, C, 1, labels=torch.empty((1, 256), dtype=torch.int32).pin_memory())
    assert e.value.status == 2


def test_host_pipeline_deadline_returns_timeout_then_recovers(monkeypatch):
    """The pipeline's bounded host wait (KM_HOST_TIMEOUT_S): a deadline far shorter than the work makes
    km_lloyd return KM_E_TIMEOUT instead of blocking; the work it enqueued still completes on the
    stream, the scratch goes back to the pool, and the next call succeeds with the same results.
    Host-side only: nothing on the GPU waits for anything that does not come."""
    w = synth.small(B=2, N=200000, d=128, K=256, dtype="f16", ncomp=256, seed=47)
    X = synth.points(w)
    C0 = torch.from_numpy(synth.init_centroids(w, X)).cuda()
    Xh = pinned(X)
    lab_h = torch.empty((w.B, w.N), dtype=torch.int32).pin_memory()
    km.lib().km_set_chunk_rows(25000)  # 8 chunks per batch
    lab_ref, C_ref, _ = km.lloyd(Xh, C0, 2, labels=lab_h)
    torch.cuda.synchronize()
    lab_ref = lab_ref.clone()
    km.lib().km_release_cached()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]

    monkeypatch.setenv("KM_HOST_TIMEOUT_S", "0.000001")
    lab2 = torch.empty_like(lab_h).pin_memory()
    with pytest.raises(km.KMError) as e:
        km.lloyd(Xh, C0, 2, labels=lab2)
    assert e.value.status == 5  # KM_E_TIMEOUT
    assert b"still running" in km.lib().km_last_error()
    torch.cuda.synchronize()  # the enqueued work completes
    monkeypatch.delenv("KM_HOST_TIMEOUT_S")
    assert km.device_fault() == 0
    km.lib().km_release_cached()
    torch.cuda.synchronize()
    assert abs(torch.cuda.mem_get_info()[0] - free0) <= 8 << 20  # nothing kept beyond the pool's slack

    lab3, C3, _ = km.lloyd(Xh, C0, 2, labels=torch.empty_like(lab_h).pin_memory())
    torch.cuda.synchronize()
    assert torch.equal(lab3, lab_ref)
    torch.testing.assert_close(C3, C_ref, rtol=1e-5, atol=1e-6)
