"""km_assign_noalloc: the assignment for callers that cannot allocate device memory.

Such callers (a framework that reserved the device's memory for its own pool,
or a latency-critical loop that must not enter the allocator) get the same
kernels with their scratch in a fixed array compiled into the library.  The
test calls the entry point through the C ABI twice in a row, with different
centroids, and compares each result with km_assign's on the same inputs.
It is collected last so that a run stopping at the first failure has already
run every other test, and it passes both alone and after the other tests.
"""
import ctypes

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
import flashassign_b200 as km  # noqa: E402

pytestmark = pytest.mark.gpu


def noalloc(X, C, labels, mindist):
    B, N, d = X.shape
    K = C.shape[1]
    code = km.KM_F16 if X.dtype == torch.float16 else km.KM_F32
    return km.lib().km_assign_noalloc(ctypes.c_void_p(X.data_ptr()), ctypes.c_void_p(C.data_ptr()), B, N, K, d,
                                      code, ctypes.c_void_p(labels.data_ptr()), ctypes.c_void_p(mindist.data_ptr()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype,d", [("f16", 128), ("f16", 96), ("f32", 16), ("f32", 128), ("f16", 256),
                                     ("f16", 1024)])
def test_noalloc_matches_km_assign_on_two_calls_in_a_row(dtype, d):
    w = synth.small(B=3, N=2500, d=d, K=300, dtype=dtype, seed=777 + d)
    X = torch.from_numpy(synth.points(w)).cuda()
    C1 = torch.from_numpy(synth.init_centroids(w, X.cpu().numpy())).cuda()
    C2 = C1.flip(1).contiguous() + 0.25  # a second, different set of centroids
    for C in (C1, C2):
        ref_lab, ref_md = km.assign(X, C)
        lab = torch.full_like(ref_lab, -7)
        md = torch.full_like(ref_md, -7.0)
        assert noalloc(X, C, lab, md) == 0, km.lib().km_last_error()
        torch.cuda.synchronize()
        # same kernels on the same inputs: identical labels and distances
        assert torch.equal(lab, ref_lab)
        assert torch.equal(md, ref_md)
    assert km.device_fault() == 0


def test_noalloc_rejects_problems_above_its_fixed_scratch():
    limit = km.lib().km_assign_noalloc_limit()
    assert limit == 16 << 20
    B, K, d = 4, 32768, 128          # 2*B*K*d bytes = 32 MiB > 16 MiB (fp16)
    X = torch.zeros((B, 256, d), dtype=torch.float16, device="cuda")
    C = torch.zeros((B, K, d), dtype=torch.float32, device="cuda")
    lab = torch.empty((B, 256), dtype=torch.int32, device="cuda")
    md = torch.empty((B, 256), dtype=torch.float32, device="cuda")
    assert noalloc(X, C, lab, md) == 2  # KM_E_UNSUPPORTED, before any work is enqueued
    assert b"use km_assign" in km.lib().km_last_error()
