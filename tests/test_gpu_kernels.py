"""Parity of each CUDA kernel with the CPU oracle on small seeded inputs, through the C ABI.

Sizes span several tiles with ragged tails: point units of 256 rows, centroid
tiles of 128 columns, 16-byte row chunks; shapes at and around those edges,
plus the degenerate cases of the method (K = 1, one cluster holding every
point, empty clusters, duplicate centroids, exact distance ties).
"""
import numpy as np
import pytest

import oracle
import synth
from parity import check_centroids, check_labels, check_sort, tau_mind

torch = pytest.importorskip("torch")
import flashassign_b200 as km  # noqa: E402

pytestmark = pytest.mark.gpu


def cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_assign(X, C):
    lab, md = km.assign(cuda(X), cuda(C))
    torch.cuda.synchronize()
    assert km.device_fault() == 0
    return lab.cpu().numpy(), md.cpu().numpy()


ASSIGN_SHAPES = [
    # (B, N, K, d, dtype)
    (1, 1, 1, 128, "f16"),
    (1, 127, 2, 128, "f16"),
    (2, 128, 8, 128, "f16"),
    (1, 129, 127, 128, "f16"),
    (3, 255, 128, 128, "f16"),
    (2, 256, 129, 128, "f16"),
    (2, 257, 255, 128, "f16"),
    (3, 1000, 300, 128, "f16"),
    (2, 20000, 1000, 128, "f16"),  # four centroid tiles kept in the ring over a pair's units of one batch
    (40, 1000, 500, 128, "f16"),   # two resident tiles, reloaded as a pair's units change batch
    (2, 777, 257, 64, "f16"),
    (2, 600, 200, 96, "f16"),
    (2, 500, 100, 16, "f16"),    # below the tensor-core range: CUDA-core kernel
    (2, 300, 50, 256, "f16"),    # wide points: centroids streamed in 64-dimension chunks
    (1, 129, 127, 192, "f16"),
    (2, 1000, 300, 512, "f16"),
    (3, 257, 513, 320, "f16"),
    (2, 500, 100, 448, "f16"),
    (2, 1000, 300, 576, "f16"),  # d > 512: points and centroids streamed along d (split-D),
    (1, 257, 700, 1024, "f16"),  # ... three centroid tiles: the last pass has one
    (1, 129, 1, 640, "f16"),
    (3, 300, 513, 768, "f16"),
    (1, 513, 1024, 2048, "f16"),
    (1, 300, 60, 4096, "f16"),
    (1, 700, 2100, 4096, "f16"),  # ... 9 centroid tiles: 5 passes, the last with one tile
    (2, 300, 1500, 3072, "f16"),  # ... 6 tiles, 3 full passes, two batches
    (1, 200, 20, 1000, "f16"),   # d > 512, not a multiple of 64: CUDA-core kernel
    (1, 100, 20, 1000, "f32"),
    (1, 200, 30, 136, "f16"),    # not a multiple of 64: CUDA-core kernel
    (1, 4096, 8, 16, "f32"),     # fp32 below the tf32 tensor-core range (d % 32 != 0): CUDA cores
    (2, 129, 33, 4, "f32"),
    (1, 1, 1, 32, "f32"),        # fp32 on tf32 tensor cores: d in {32, 64, 96, 128}
    (1, 129, 127, 128, "f32"),
    (2, 257, 255, 32, "f32"),
    (3, 255, 129, 64, "f32"),
    (2, 777, 257, 96, "f32"),
    (2, 1000, 300, 128, "f32"),
    (2, 1000, 513, 128, "f32"),
    (1, 300, 50, 160, "f32"),    # above it
]


@pytest.mark.parametrize("B,N,K,d,dt", ASSIGN_SHAPES)
def test_assign_matches_oracle(B, N, K, d, dt):
    w = synth.small(B=B, N=N, d=d, K=K, dtype=dt, ncomp=max(1, K // 2), sigma=0.3, seed=1000 + N + K + d)
    X = synth.points(w)
    C = synth.init_centroids(w, X) if K <= N else np.random.default_rng(1).standard_normal((B, K, d)).astype(
        np.float32)
    lab, md = run_assign(X, C)
    check_labels(X, C, lab, md)


@pytest.mark.parametrize("dt,d", [("f16", 128), ("f16", 256), ("f32", 16), ("f32", 128)])
def test_assign_ties_go_to_the_lowest_index(dt, d):
    # integer coordinates and duplicate centroids give exact ties in every precision
    rng = np.random.default_rng(11)
    B, N, K = 2, 700, 260
    npdt = np.float16 if dt == "f16" else np.float32
    X = rng.integers(-2, 3, (B, N, d)).astype(npdt)
    base = rng.integers(-2, 3, (B, 40, d)).astype(np.float32)
    C = base[:, rng.integers(0, 40, K)]  # many duplicates, at indices far apart
    lab, md = run_assign(X, C)
    ref, d1, d2 = oracle.assign(X, C)
    assert np.array_equal(lab, ref)
    assert np.array_equal(md, d1.astype(np.float32))


def test_fp32_tensor_cores_resolve_clear_points_and_list_the_rest():
    # well-separated mixture: almost every point is resolved by the tf32 tensor cores
    w = synth.small(B=2, N=4000, d=128, K=300, dtype="f32", ncomp=150, sigma=0.3, seed=77)
    X = synth.points(w)
    C = synth.init_centroids(w, X)
    km.assign_rescans()
    lab, md = run_assign(X, C)
    listed = km.assign_rescans()
    check_labels(X, C, lab, md)
    assert listed < 0.05 * w.B * w.N, f"{listed} of {w.B * w.N} points needed the exact re-scan"
    # identical centroids: every score ties, every point goes to the re-scan and to centroid 0
    C_same = np.repeat(C[:, :1], 300, axis=1)
    lab, md = run_assign(X, C_same)
    assert km.assign_rescans() == w.B * w.N
    assert (lab == 0).all()
    check_labels(X, C_same, lab, md)


def test_fp32_tensor_cores_exact_where_the_gap_is_clear_far_from_the_origin():
    # points and centroids offset from the origin: ||x||^2 and ||c||^2 dwarf the distances, so the
    # expansion cancels; labels must still be exact wherever the relative top-2 gap is >= 1e-5
    rng = np.random.default_rng(78)
    B, N, K, d = 2, 3000, 200, 64
    centres = rng.standard_normal((B, 40, d)) + 4.0
    X = (centres[:, rng.integers(0, 40, N)] + 0.05 * rng.standard_normal((B, N, d))).astype(np.float32)
    C = X[:, rng.choice(N, K, replace=False)].copy()
    km.assign_rescans()
    lab, md = run_assign(X, C)
    km.assign_rescans()
    check_labels(X, C, lab, md)


FP16_TC_WIDTHS = [64, 128, 256, 512, 1024, 4096]  # the d <= 128, wide and split-D tensor-core kernels


def _far_mixture(rng, B, N, ncomp, d, offset, spread, sigma):
    """Points of a Gaussian mixture whose centres sit at `offset` + spread * N(0,1) per coordinate."""
    centres = offset + spread * rng.standard_normal((B, ncomp, d))
    comp = rng.integers(0, ncomp, (B, N))
    X = (np.take_along_axis(centres, comp[..., None], axis=1) + sigma * rng.standard_normal((B, N, d)))
    return X.astype(np.float16), centres


@pytest.mark.parametrize("d", FP16_TC_WIDTHS)
def test_fp16_large_norms_fold_exactly(d):
    # ||c||^2 of several million, far past what 16 unit-weight fp16 pieces of -||c||^2/2 can hold
    # (~2.1e6), on data the tensor cores can certify: for d <= 128 (certified from the best score)
    # points spread widely around their centres, for wider points (certified from the best two
    # scores) tight clusters far apart; almost every label comes from the tensor cores
    rng = np.random.default_rng(80 + d)
    B, N, K = 2, (1000 if d <= 512 else 300), (300 if d <= 512 else 60)
    offset = float(np.sqrt(6e6 / d))
    spread, sigma = (offset / 2, offset / 4) if d <= 128 else (offset / 10, 1.0)
    X, centres = _far_mixture(rng, B, N, K, d, offset, spread, sigma)
    C = (centres + 0.5 * rng.standard_normal(centres.shape)).astype(np.float32)
    assert (np.square(C.astype(np.float16).astype(np.float64)).sum(-1) > 4e6).all()
    km.assign_rescans()
    lab, md = run_assign(X, C)
    listed = km.assign_rescans()
    check_labels(X, C, lab, md)
    assert listed < 0.05 * B * N, f"{listed} of {B * N} points went to the exact re-scan"


@pytest.mark.parametrize("d", [128, 1024])
def test_fp16_norms_beyond_the_folded_range_are_rescanned_exactly(d):
    # ||c||^2 / 2 above the folded term's ~1.7e10: every point of the batch goes to the exact
    # CUDA-core re-scan, none gets a truncated score
    rng = np.random.default_rng(90 + d)
    B, N, K = 2, 400, 50
    offset = float(np.sqrt(6e10 / d))
    X, centres = _far_mixture(rng, B, N, K, d, offset, offset / 10, offset / 100)
    C = (centres + offset / 100 * rng.standard_normal(centres.shape)).astype(np.float32)
    assert (np.square(C.astype(np.float16).astype(np.float64)).sum(-1) > 3.5e10).all()
    km.assign_rescans()
    lab, md = run_assign(X, C)
    assert km.assign_rescans() == B * N
    check_labels(X, C, lab, md)


@pytest.mark.parametrize("d", FP16_TC_WIDTHS)
def test_fp16_tensor_cores_exact_where_the_gap_is_clear_far_from_the_origin(d):
    # the fp16 twin of the fp32 test above: ||x||^2 and ||c||^2 dwarf the distances, so the
    # expansion cancels; labels must be exact wherever the relative top-2 gap is >= 1e-3
    rng = np.random.default_rng(78 + d)
    B, N, K = 2, (3000 if d <= 512 else 800), (200 if d <= 512 else 80)
    centres = rng.standard_normal((B, 40, d)) + 4.0
    X = (centres[:, rng.integers(0, 40, N)] + 0.05 * rng.standard_normal((B, N, d))).astype(np.float16)
    C = X[:, rng.choice(N, K, replace=False)].astype(np.float32)
    km.assign_rescans()
    lab, md = run_assign(X, C)
    listed = km.assign_rescans()
    check_labels(X, C, lab, md)
    print(f"d={d}: {listed} of {B * N} points re-scanned")


@pytest.mark.parametrize("d", [128, 256, 1024])
def test_fp16_duplicate_centroids_resolve_to_the_lowest_index(d):
    # every centroid twice, 100 columns apart (some pairs in one 32-column group, most not): the
    # duplicates' scores are equal bit for bit, and the label must be the lower index as in the
    # oracle, whether the tensor cores certify the point or the exact re-scan takes it
    rng = np.random.default_rng(31 + d)
    B, N, K = 2, 2000, 200
    X = rng.standard_normal((B, N, d)).astype(np.float16)
    base = rng.standard_normal((B, K // 2, d)).astype(np.float32)
    C = np.concatenate([base, base], axis=1)
    C[:, 1::7] = C[:, 0::7][:, :C[:, 1::7].shape[1]]  # and some neighbours equal inside a group
    lab, md = run_assign(X, C)
    ref, d1, d2 = oracle.assign(X, C)
    assert np.array_equal(lab, ref)
    check_labels(X, C, lab, md)


def test_rescan_of_many_batches_takes_smaller_clusters():
    # 40 batches: clusters of 16 CTAs for every batch would not all fit on the device at once, so the
    # re-scan takes clusters of 8; centroid norms beyond the folded term's range send every point of
    # every batch to it
    rng = np.random.default_rng(91)
    B, N, K, d = 40, 200, 50, 128
    offset = float(np.sqrt(6e10 / d))
    X, centres = _far_mixture(rng, B, N, K, d, offset, offset / 10, offset / 100)
    C = (centres + offset / 100 * rng.standard_normal(centres.shape)).astype(np.float32)
    km.assign_rescans()
    lab, md = run_assign(X, C)
    assert km.assign_rescans() == B * N
    check_labels(X, C, lab, md)


def test_assign_single_centroid_and_far_centroids():
    rng = np.random.default_rng(12)
    X = rng.standard_normal((2, 300, 128)).astype(np.float16)
    C = rng.standard_normal((2, 1, 128)).astype(np.float32)
    lab, md = run_assign(X, C)
    assert (lab == 0).all()
    check_labels(X, C, lab, md)


@pytest.mark.parametrize("case", ["random", "all_equal", "k1", "sorted", "skewed", "big_k", "ragged",
                                  "one_pass_max", "one_pass_tiles", "one_pass_tail", "k4096", "long_small_k",
                                  "small_max", "small_odd", "small_one", "small_33", "small_reversed", "just_over",
                                  "cluster_13", "cluster_tail_one", "top_bin"])
def test_sort_is_bit_exact(case):
    rng = np.random.default_rng(13)
    B, N, K = 3, 5000, 1024
    if case == "random":
        lab = rng.integers(0, K, (B, N))
    elif case == "all_equal":
        lab = np.full((B, N), 517)
    elif case == "k1":
        K = 1
        lab = np.zeros((B, N))
    elif case == "sorted":
        lab = np.sort(rng.integers(0, K, (B, N)), axis=1)
    elif case == "skewed":
        lab = np.minimum(rng.zipf(1.2, (B, N)) - 1, K - 1)
    elif case == "big_k":
        K = 65536
        lab = rng.integers(0, K, (B, N))
    elif case == "ragged":
        B, N, K = 2, 2049, 3000  # one key past a 2048-key tile; 12-bit keys
        lab = rng.integers(0, K, (B, N))
    elif case == "one_pass_max":
        B, N, K = 2, 9000, 2048  # the largest single-pass label range
        lab = rng.integers(0, K, (B, N))
    elif case == "one_pass_tiles":
        B, N, K = 2, 70000, 2000  # 18 tiles of 4096 keys, the last one ragged
        lab = rng.integers(0, K, (B, N))
    elif case == "long_small_k":
        B, N, K = 1, 300000, 1000  # more tiles than the single pass takes: two 5-bit radix passes
        lab = rng.integers(0, K, (B, N))
    elif case == "one_pass_tail":
        B, N, K = 3, 4097, 5  # one key past a 4096-key tile, a few labels
        lab = rng.integers(0, K, (B, N))
    # single batches at and around 2^16 points
    elif case == "small_max":
        B, N, K = 2, 65536, 1024
        lab = rng.integers(0, K, (B, N))
    elif case == "small_odd":
        B, N, K = 3, 65535, 1000  # odd length, skewed labels
        lab = np.minimum(rng.zipf(1.2, (B, N)) - 1, K - 1)
    elif case == "small_one":
        B, N, K = 2, 1, 1
        lab = np.zeros((B, N))
    elif case == "small_33":
        B, N, K = 2, 33, 7  # one full warp group and one lane of the next
        lab = rng.integers(0, K, (B, N))
    elif case == "small_reversed":
        B, N, K = 1, 40000, 1024
        lab = np.sort(rng.integers(0, K, (B, N)), axis=1)[:, ::-1]
    elif case == "just_over":
        B, N, K = 1, 65537, 1024  # one point past 2^16
        lab = rng.integers(0, K, (B, N))
    # single-launch cluster sort: one CTA per 4096 points of a batch
    elif case == "cluster_13":
        B, N, K = 2, 50000, 600  # a cluster of 13 CTAs, 10-bit labels not filling their range
        lab = rng.integers(0, K, (B, N))
    elif case == "cluster_tail_one":
        B, N, K = 3, 8193, 1024  # the third CTA holds one point
        lab = rng.integers(0, K, (B, N))
    elif case == "top_bin":
        B, N, K = 2, 65536, 1024  # nearly every label in the last bin, a few in the first
        lab = np.full((B, N), K - 1)
        lab[:, rng.integers(0, N, 100)] = 0
    else:
        B, N, K = 2, 20000, 4096  # two 6-bit passes
        lab = np.minimum(rng.zipf(1.1, (B, N)) - 1, K - 1)
    lab = lab.astype(np.int32)
    sidx, counts, offsets = km.sort_labels(cuda(lab), K)
    torch.cuda.synchronize()
    check_sort(lab, K, sidx.cpu().numpy(), counts.cpu().numpy(), offsets.cpu().numpy())


@pytest.mark.parametrize("B,N,K,d,dt,case", [
    (2, 1000, 40, 128, "f16", "random"),
    (2, 5000, 300, 128, "f16", "zipf"),
    (1, 3000, 7, 128, "f16", "one_cluster"),
    (2, 2000, 500, 128, "f16", "empty"),
    (1, 4096, 8, 16, "f32", "random"),
    (2, 1500, 100, 128, "f32", "zipf"),
    (2, 999, 64, 64, "f16", "random"),
    (1, 700, 30, 512, "f32", "random"),
    (1, 700, 30, 512, "f16", "zipf"),
    (1, 700, 30, 2048, "f16", "random"),   # rows over 1 KB: split into 1 KB slices
    (1, 500, 20, 1000, "f32", "zipf"),     # ... with a narrower last slice
    (2, 600, 40, 600, "f32", "empty"),
    (1, 900, 25, 4096, "f16", "one_cluster"),
])
def test_update_matches_oracle(B, N, K, d, dt, case):
    rng = np.random.default_rng(14)
    w = synth.small(B=B, N=N, d=d, K=K, dtype=dt, seed=77 + K)
    X = synth.points(w)
    if case == "random":
        lab = rng.integers(0, K, (B, N))
    elif case == "zipf":
        lab = np.minimum(rng.zipf(1.2, (B, N)) - 1, K - 1)
    elif case == "one_cluster":
        lab = np.full((B, N), 3)
    else:
        lab = rng.integers(0, K // 3, (B, N)) * 3  # two thirds of the clusters empty
    lab = lab.astype(np.int32)
    C_prev = rng.standard_normal((B, K, d)).astype(np.float32)
    C_out, sums, counts = km.update(cuda(X), cuda(lab), cuda(C_prev))
    torch.cuda.synchronize()
    check_centroids(X, lab, C_prev, C_out.cpu().numpy(), counts.cpu().numpy(), sums.cpu().numpy())


@pytest.mark.parametrize("B,N,K,d,dt", [(2, 3000, 50, 128, "f16"), (1, 4096, 8, 16, "f32"), (2, 1000, 300, 64, "f16"),
                                        (2, 3000, 50, 128, "f32"), (1, 2000, 257, 32, "f32"),
                                        (1, 3000, 300, 512, "f16"), (2, 1000, 100, 256, "f16"),
                                        (1, 1500, 100, 1024, "f16"), (1, 800, 40, 4096, "f16"),
                                        (1, 1500, 1100, 2048, "f16")])
def test_lloyd_lockstep_with_oracle(B, N, K, d, dt):
    """Each iteration: the oracle takes the GPU's centroids and checks that iteration's labels and update."""
    w = synth.small(B=B, N=N, d=d, K=K, dtype=dt, ncomp=K, sigma=0.3, seed=5 + K)
    X = synth.points(w)
    C = synth.init_centroids(w, X)
    Xg = cuda(X)
    near = 0
    for t in range(5):
        lab, C_next, obj = km.lloyd(Xg, cuda(C), 1)
        torch.cuda.synchronize()
        lab, C_next, obj = lab.cpu().numpy(), C_next.cpu().numpy(), obj.cpu().numpy()
        near += check_labels(X, C, lab)
        check_sort(lab, K, *[a.cpu().numpy() for a in km.sort_labels(cuda(lab), K)])
        check_centroids(X, lab, C, C_next)
        _, d1, _ = oracle.assign(X, C)
        # the objective sums the points' minimum distances: within the sum of their rounding bounds
        chat = oracle.round_centroids(C, oracle.F16 if dt == "f16" else oracle.F32)
        cg = np.take_along_axis(chat, lab[..., None].astype(np.int64), axis=1)
        scale = (X.astype(np.float64) ** 2).sum(-1) + (cg.astype(np.float64) ** 2).sum(-1)
        ref = d1.sum(axis=1)
        assert (np.abs(obj[0] - ref) <= 1e-4 * np.abs(ref) + tau_mind(d) * scale.sum(axis=1)).all(), (obj[0], ref)
        C = C_next
    assert km.device_fault() == 0


def test_lloyd_many_iterations_equal_one_at_a_time():
    w = synth.small(B=2, N=2000, d=128, K=64, dtype="f16", seed=21)
    X = synth.points(w)
    C0 = synth.init_centroids(w, X)
    Xg = cuda(X)
    lab6, C6, obj6 = km.lloyd(Xg, cuda(C0), 6)
    C = cuda(C0)
    objs = []
    for t in range(6):
        lab1, C, o = km.lloyd(Xg, C, 1)
        objs.append(o)
    torch.cuda.synchronize()
    # resuming from saved centroids reproduces the run (sums may differ in the last bits
    # through the order of boundary atomics, hence the tolerance)
    np.testing.assert_allclose(C6.cpu().numpy(), C.cpu().numpy(), rtol=1e-5, atol=1e-5)
    assert (lab6.cpu().numpy() == lab1.cpu().numpy()).mean() > 0.999
    np.testing.assert_allclose(obj6.cpu().numpy(), torch.cat(objs).cpu().numpy(), rtol=1e-5)


@pytest.mark.parametrize("B,N,K,launches", [(32, 65536, 1024, 1), (3, 4097, 8, 1), (2, 65537, 1024, 6),
                                            (2, 20000, 2048, 6)])
def test_sort_path_by_shape(B, N, K, launches):
    """Batches of at most 65,536 labels below 1024 are sorted in one launch (a thread-block cluster per
    batch); longer batches or wider labels take the radix passes (a histogram and a scatter per pass)
    plus the boundary and count kernels.  Both give the oracle's bit-exact result."""
    rng = np.random.default_rng(B * N + K)
    lab = rng.integers(0, K, (B, N)).astype(np.int32)
    g = cuda(lab)
    km.sort_labels(g, K)
    torch.cuda.synchronize()
    km.trace_enable(True)
    try:
        km.trace_read()
        sidx, counts, offsets = km.sort_labels(g, K)
        torch.cuda.synchronize()
        rec = km.trace_read()
    finally:
        km.trace_enable(False)
    assert rec["sort"][1] == launches
    check_sort(lab, K, sidx.cpu().numpy(), counts.cpu().numpy(), offsets.cpu().numpy())


def test_labels_counts_and_sort_are_deterministic():
    w = synth.small(B=2, N=5000, d=128, K=200, dtype="f16", seed=22)
    X = cuda(synth.points(w))
    C = cuda(synth.init_centroids(w, X.cpu().numpy()))
    outs = []
    for _ in range(3):
        lab, md = km.assign(X, C)
        sidx, counts, offs = km.sort_labels(lab, w.K)
        outs.append([t.cpu().numpy() for t in (lab, md, sidx, counts, offs)])
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert np.array_equal(a, b)


def test_objective_never_increases_beyond_rounding():
    w = synth.small(B=2, N=4000, d=128, K=100, dtype="f16", ncomp=100, seed=23)
    X = synth.points(w)
    C0 = synth.init_centroids(w, X)
    _, _, obj = km.lloyd(cuda(X), cuda(C0), 12)
    obj = obj.cpu().numpy().astype(np.float64)
    # fp16 rounding of the centroids can add a little; it must stay tiny relative to J
    assert (np.diff(obj, axis=0) <= 1e-3 * obj[:-1]).all()
    assert (obj[-1] < obj[0]).all()


def test_injected_allocation_failure_is_reported_and_leaks_nothing(monkeypatch):
    w = synth.small(B=1, N=1000, d=128, K=50, dtype="f16", seed=24)
    X = cuda(synth.points(w))
    C = cuda(synth.init_centroids(w, X.cpu().numpy()))
    km.lloyd(X, C, 1)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    monkeypatch.setenv("KM_FAULT", "alloc")
    with pytest.raises(km.KMError) as e:
        km.lloyd(X, C, 2)
    assert e.value.status == 3
    monkeypatch.setenv("KM_FAULT", "launch")
    with pytest.raises(km.KMError) as e:
        km.assign(X, C)
    assert e.value.status == 4
    monkeypatch.delenv("KM_FAULT")
    torch.cuda.synchronize()
    assert abs(torch.cuda.mem_get_info()[0] - free0) < (64 << 20)
    km.lloyd(X, C, 1)  # still works
    torch.cuda.synchronize()


# ---- the baselines the method replaces (measurement only) ----

@pytest.mark.parametrize("B,N,K,d", [(2, 1000, 300, 128), (1, 129, 127, 64), (2, 257, 255, 96), (3, 511, 513, 128),
                                     (4, 20000, 1000, 128)])  # resident centroid tiles over several units per pair
def test_dense_assign_baseline_matches_the_fused_kernel_and_the_oracle(B, N, K, d):
    w = synth.small(B=B, N=N, d=d, K=K, dtype="f16", ncomp=max(1, K // 2), sigma=0.3, seed=2000 + N + K)
    X = synth.points(w)
    C = synth.init_centroids(w, X) if K <= N else np.random.default_rng(2).standard_normal((B, K, d)).astype(
        np.float32)
    lab_d, md_d = km.assign_dense(cuda(X), cuda(C))
    lab_f, md_f = km.assign(cuda(X), cuda(C))
    torch.cuda.synchronize()
    assert km.device_fault() == 0
    lab_d, md_d = lab_d.cpu().numpy(), md_d.cpu().numpy()
    # the same scores from the same MMAs, reduced on chip or read back: identical results
    assert np.array_equal(lab_d, lab_f.cpu().numpy())
    assert np.array_equal(md_d, md_f.cpu().numpy())
    check_labels(X, C, lab_d, md_d)


def test_dense_assign_baseline_rejects_shapes_outside_the_tensor_core_range():
    X = torch.zeros((1, 64, 16), dtype=torch.float16, device="cuda")
    C = torch.zeros((1, 4, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(km.KMError) as e:
        km.assign_dense(X, C)
    assert e.value.status == 2


@pytest.mark.parametrize("B,N,K,d,dt", [(2, 3000, 100, 128, "f16"), (1, 4096, 8, 16, "f32"), (2, 2000, 500, 64, "f16")])
def test_scatter_update_baseline_matches_the_oracle(B, N, K, d, dt):
    w = synth.small(B=B, N=N, d=d, K=K, dtype=dt, ncomp=K, sigma=0.3, seed=3000 + N + K)
    X = synth.points(w)
    C = synth.init_centroids(w, X)
    lab, _ = run_assign(X, C)
    C_s, sums_s, counts_s = km.update_scatter(cuda(X), cuda(lab), cuda(C))
    C_u, sums_u, counts_u = km.update(cuda(X), cuda(lab), cuda(C))
    torch.cuda.synchronize()
    assert torch.equal(counts_s, counts_u)
    check_centroids(X, lab, C, C_s.cpu().numpy(), counts_s.cpu().numpy())


# ---- convergence-controlled iteration (device-side stop) ----

def _shift(Ca, Cb):
    return ((np.asarray(Ca, np.float64) - np.asarray(Cb, np.float64)) ** 2).sum(axis=(1, 2))


@pytest.mark.parametrize("dt,d,K", [("f16", 128, 40), ("f32", 128, 40), ("f32", 16, 12), ("f16", 256, 40),
                                    ("f16", 1024, 40)])
def test_lloyd_tol_stops_when_the_centroids_settle_and_equals_plain_iterations(dt, d, K):
    w = synth.small(B=3, N=3000, d=d, K=K, dtype=dt, ncomp=K, sigma=0.2, seed=4000 + d + K)
    X = synth.points(w)
    C0 = cuda(synth.init_centroids(w, X))
    Xg = cuda(X)
    tol = 1e-9  # above the last-bit wander of sums combined by atomics, far below any real move
    lab, C, obj, n = km.lloyd_tol(Xg, C0, 60, tol)
    torch.cuda.synchronize()
    t = int(n.item())
    assert 1 <= t < 60, f"not settled within 60 iterations ({t})"
    lab_p, C_p, obj_p = km.lloyd(Xg, C0, t)
    torch.cuda.synchronize()
    # the same kernels in the same order as t plain iterations (up to the order of fp32 atomics)
    assert (lab == lab_p).float().mean().item() > 0.9999
    torch.testing.assert_close(C, C_p, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(obj[:t], obj_p, rtol=1e-5, atol=0)
    assert torch.isnan(obj[t:]).all()  # rows past the stop are not written
    # the stop was earned: one more iteration moves the centroids by at most tol
    _, C_next, _ = km.lloyd(Xg, C, 1)
    torch.cuda.synchronize()
    assert (_shift(C_next.cpu().numpy(), C.cpu().numpy()) <= 10 * tol).all()
    assert km.device_fault() == 0


@pytest.mark.parametrize("dt,d,K", [("f16", 128, 60), ("f32", 64, 40), ("f16", 1024, 30)])
def test_lloyd_tol_stops_where_the_oracle_does_in_lock_step(dt, d, K):
    """The stopping rule against the oracle: iteration by iteration the oracle takes the GPU's
    centroids, checks that iteration's labels and update, and computes the shift of its own
    update; the loop must stop after the first iteration whose shift is within tol in every
    batch (oracle.lloyd_tol's rule), for a tol chosen away from every shift of the run."""
    w = synth.small(B=2, N=3000, d=d, K=K, dtype=dt, ncomp=K, sigma=0.3, seed=4200 + d + K)
    X = synth.points(w)
    C0 = synth.init_centroids(w, X)
    Xg = cuda(X)
    Cs, shifts, labs = [C0], [], []
    for t in range(12):
        lab, C_next, _ = km.lloyd(Xg, cuda(Cs[-1]), 1)
        torch.cuda.synchronize()
        lab, C_next = lab.cpu().numpy(), C_next.cpu().numpy()
        check_labels(X, Cs[-1], lab)
        C_ref = check_centroids(X, lab, Cs[-1], C_next)
        shifts.append(_shift(C_ref, Cs[-1]))  # the oracle's update of the GPU's centroids
        labs.append(lab)
        Cs.append(C_next)
    S = np.array([s.max() for s in shifts])  # a batch stops the loop only with every other batch
    # a tolerance a factor of 3 away from every shift up to the stop it causes, stopping after >= 2 iterations
    best = None
    for i in range(1, len(S) - 1):
        tol = float(np.sqrt(S[i] * S[i + 1])) if S[i + 1] > 0 else S[i] / 9
        T = next((t + 1 for t, s in enumerate(S) if s <= tol), None)
        if T is None or T < 2 or tol <= 0:
            continue
        margin = min(abs(np.log(max(S[t], 1e-300) / tol)) for t in range(T))
        if best is None or margin > best[2]:
            best = (tol, T, margin)
    assert best is not None and best[2] > np.log(3), f"no well-separated tolerance in shifts {S}"
    tol, T, _ = best
    lab_g, C_g, obj_g, n = km.lloyd_tol(Xg, cuda(C0), 12, tol)
    torch.cuda.synchronize()
    assert int(n.item()) == T, (int(n.item()), T, S, tol)
    # its last labels match the oracle from the centroids before them, and its centroids those
    # of the replay (checked against the oracle above; the two runs may differ in the last bits,
    # where fp32 atomics add partial sums in another order)
    check_labels(X, Cs[T - 1], lab_g.cpu().numpy())
    np.testing.assert_allclose(C_g.cpu().numpy(), Cs[T], rtol=1e-4, atol=1e-6)
    assert km.device_fault() == 0


def test_lloyd_tol_applies_the_shift_rule_and_the_iteration_cap():
    w = synth.small(B=2, N=4000, d=64, K=60, dtype="f16", ncomp=60, sigma=0.3, seed=4101)
    X = synth.points(w)
    C0 = cuda(synth.init_centroids(w, X))
    Xg = cuda(X)
    runs = [km.lloyd(Xg, C0, t)[1].cpu().numpy() for t in range(1, 9)]  # C after t iterations
    shifts = [_shift(runs[0], C0.cpu().numpy())] + [_shift(runs[t], runs[t - 1]) for t in range(1, 8)]
    # a tolerance between two of the per-iteration shifts, away from either (the device sums in another order)
    vals = sorted({float(s.max()) for s in shifts})
    tol = 0.5 * (vals[len(vals) // 2 - 1] + vals[len(vals) // 2])
    _, C, _, n = km.lloyd_tol(Xg, C0, 8, tol)
    torch.cuda.synchronize()
    t = int(n.item())
    # stopped after the first iteration whose shift is within tol in every batch
    first = next((i + 1 for i, s in enumerate(shifts) if (s <= tol).all()), 8)
    assert t == first
    assert np.array_equal(C.cpu().numpy(), runs[t - 1])
    # the cap: two iterations at most
    _, _, _, n2 = km.lloyd_tol(Xg, C0, 2, 0.0)
    torch.cuda.synchronize()
    assert int(n2.item()) == 2


def test_lloyd_tol_rejects_bad_arguments():
    X = torch.zeros((1, 256, 64), dtype=torch.float16, device="cuda")
    C = torch.zeros((1, 4, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(km.KMError) as e:
        km.lloyd_tol(X, C, 5, -1.0)
    assert e.value.status == 1
    with pytest.raises(km.KMError) as e:
        km.lloyd_tol(X.cpu().pin_memory(), C, 5, 0.0)
    assert e.value.status == 2


def test_scratch_pool_keeps_memory_until_released():
    # the dense baseline takes a 256 MiB score matrix as scratch; the library's pool keeps it after the call
    w = synth.small(B=1, N=65536, d=128, K=1024, dtype="f16", seed=25)
    X = cuda(synth.points(w))
    C = cuda(synth.init_centroids(w, X.cpu().numpy()))
    km.assign_dense(X, C)
    torch.cuda.synchronize()
    held = torch.cuda.mem_get_info()[0]
    km.assign_dense(X, C)  # served from the pool: no new device memory
    torch.cuda.synchronize()
    assert abs(torch.cuda.mem_get_info()[0] - held) < (32 << 20)
    km.check("km_release_cached", km.lib().km_release_cached())
    assert torch.cuda.mem_get_info()[0] - held > (200 << 20)


def test_concurrent_host_threads_on_their_own_streams_match_sequential_calls():
    """The entry points are reentrant: host threads calling them at once, each on its own stream,
    share the library's caches and scratch pool and get the results of the same calls made one by one."""
    import threading
    shapes = [(2, 3000, 100, 128, "f16"), (1, 2000, 300, 256, "f16"), (2, 1500, 50, 64, "f32"),
              (1, 1000, 40, 1024, "f16")]
    inputs = []
    for i, (B, N, K, d, dt) in enumerate(shapes):
        w = synth.small(B=B, N=N, d=d, K=K, dtype=dt, ncomp=K, sigma=0.3, seed=9000 + i)
        X = synth.points(w)
        inputs.append((cuda(X), cuda(synth.init_centroids(w, X))))
    ref = []
    for X, C in inputs:
        lab, C_next, _ = km.lloyd(X, C, 3)
        torch.cuda.synchronize()
        ref.append((lab.cpu(), C_next.cpu()))
    out = [None] * len(inputs)
    errors = []

    def work(i):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                X, C = inputs[i]
                for _ in range(4):
                    lab, C_next, _ = km.lloyd(X, C, 3, stream=s)
                s.synchronize()
                out[i] = (lab.cpu(), C_next.cpu())
        except Exception as e:  # reported below, on the test's thread
            errors.append(e)

    threads = [threading.Thread(target=work, args=(i,)) for i in range(len(inputs))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    assert km.device_fault() == 0
    for (lab, C_next), (ref_lab, ref_C) in zip(out, ref):
        # the same kernels on the same inputs; only the order of fp32 atomics may differ
        assert (lab == ref_lab).float().mean().item() > 0.999
        torch.testing.assert_close(C_next, ref_C, rtol=1e-5, atol=1e-6)
