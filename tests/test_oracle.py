"""Pins for the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute: exhaustive
enumeration on tiny inputs, hand-worked examples (tests/golden), library
routines it does not use (numpy's binary16 conversion, scipy's cdist, numpy's
stable argsort and mean), and invariants of Lloyd's iteration (the update is
the minimiser of the cost for fixed labels; the objective never increases).
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy.spatial.distance import cdist

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


# ---- binary16 codec -----------------------------------------------------------

def test_f16_decode_every_pattern_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_decode(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.signbit(ours[0x8000]) and not np.signbit(ours[0])


def test_f16_encode_rounds_to_nearest_even_like_numpy():
    rng = np.random.default_rng(7)
    edge = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6,
            2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -25, 2.0 ** -26, 5 * 2.0 ** -26, 2.0 ** -14,
            2.0 ** -14 - 2.0 ** -25, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 2048 + 1, 2048 + 3,
            np.inf, -np.inf]
    x = np.concatenate([np.array(edge),
                        rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 5, 20000),
                        rng.integers(-4096, 4096, 2000) * 0.5])
    ours = oracle.f16_encode(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


# ---- assignment ---------------------------------------------------------------

def _brute_force_labels(X, C):
    """Lexicographically first labelling minimising the total squared distance,
    by enumerating all K^N labellings with exact integer arithmetic."""
    N, K = X.shape[0], C.shape[0]
    best, best_lab = None, None
    for lab in itertools.product(range(K), repeat=N):  # lexicographic order
        tot = sum(int(((X[i] - C[lab[i]]) ** 2).sum()) for i in range(N))
        if best is None or tot < best:
            best, best_lab = tot, lab
    return np.array(best_lab), best


@pytest.mark.parametrize("seed", range(25))
def test_assign_equals_exhaustive_enumeration_on_tiny_integer_inputs(seed):
    rng = np.random.default_rng(seed)
    N, K, d = int(rng.integers(1, 7)), int(rng.integers(1, 4)), int(rng.integers(1, 3))
    X = rng.integers(-3, 4, size=(N, d))  # small integers: many exact ties
    C = rng.integers(-3, 4, size=(K, d))
    want, total = _brute_force_labels(X, C)
    for dt in (np.float32, np.float16):
        lab, d1, _ = oracle.assign(X[None].astype(dt), C[None].astype(np.float32))
        assert np.array_equal(lab[0], want)
        assert d1.sum() == total


@pytest.mark.parametrize("dt", [np.float32, np.float16])
def test_assign_matches_scipy_cdist_argmin(dt):
    rng = np.random.default_rng(3)
    B, N, K, d = 3, 300, 17, 24
    X = rng.standard_normal((B, N, d)).astype(dt)
    C = rng.standard_normal((B, K, d)).astype(np.float32)
    lab, d1, d2 = oracle.assign(X, C)
    for b in range(B):
        Cb = C[b].astype(dt).astype(np.float64)  # the assignment sees C in X's dtype
        D = cdist(X[b].astype(np.float64), Cb, "sqeuclidean")
        srt = np.sort(D, axis=1)
        np.testing.assert_allclose(d1[b], srt[:, 0], rtol=1e-12)
        np.testing.assert_allclose(d2[b], srt[:, 1], rtol=1e-12)
        clear = (srt[:, 1] - srt[:, 0]) > 1e-9 * srt[:, 1]
        assert np.array_equal(lab[b][clear], D.argmin(axis=1)[clear])


def test_assign_single_centroid_is_plain_distance():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((2, 50, 8)).astype(np.float32)
    C = rng.standard_normal((2, 1, 8)).astype(np.float32)
    lab, d1, d2 = oracle.assign(X, C)
    assert (lab == 0).all() and np.isinf(d2).all()
    for b in range(2):
        np.testing.assert_allclose(d1[b], cdist(X[b].astype(np.float64), C[b].astype(np.float64),
                                                "sqeuclidean")[:, 0], rtol=1e-13)


def test_assign_sampled_rows_equal_full_rows():
    w = synth.small(B=2, N=400, d=32, K=9, dtype="f16")
    X = synth.points(w)
    C = synth.init_centroids(w, X)
    lab, d1, d2 = oracle.assign(X, C)
    rows = np.array([0, 5, 399, 400, 799, 123])
    ls, s1, s2 = oracle.assign(X, C, rows=rows)
    assert np.array_equal(ls, lab.reshape(-1)[rows])
    assert np.array_equal(s1, d1.reshape(-1)[rows]) and np.array_equal(s2, d2.reshape(-1)[rows])


# ---- argsort ------------------------------------------------------------------

@pytest.mark.parametrize("case", ["random", "all_equal", "k1", "sorted", "reverse", "skewed"])
def test_sort_equals_stable_argsort(case):
    rng = np.random.default_rng(5)
    B, N, K = 3, 1000, 37
    if case == "random":
        lab = rng.integers(0, K, (B, N))
    elif case == "all_equal":
        lab = np.full((B, N), 11)
    elif case == "k1":
        K = 1
        lab = np.zeros((B, N), dtype=np.int64)
    elif case == "sorted":
        lab = np.sort(rng.integers(0, K, (B, N)), axis=1)
    elif case == "reverse":
        lab = np.sort(rng.integers(0, K, (B, N)), axis=1)[:, ::-1]
    else:
        lab = np.minimum(rng.zipf(1.5, (B, N)) - 1, K - 1)
    lab = lab.astype(np.int32)
    sidx, counts, offsets = oracle.sort_labels(lab, K)
    for b in range(B):
        assert np.array_equal(sidx[b], np.argsort(lab[b], kind="stable"))
        assert np.array_equal(counts[b], np.bincount(lab[b], minlength=K))
        assert np.array_equal(offsets[b], np.concatenate([[0], np.cumsum(np.bincount(lab[b], minlength=K))]))


def test_sort_rejects_out_of_range_labels():
    with pytest.raises(ValueError):
        oracle.sort_labels(np.array([[0, 3]], dtype=np.int32), 3)


# ---- update -------------------------------------------------------------------

@pytest.mark.parametrize("dt", [np.float32, np.float16])
def test_update_is_the_member_mean_and_empty_clusters_keep_their_centroid(dt):
    rng = np.random.default_rng(6)
    B, N, K, d = 2, 500, 30, 16
    X = (rng.standard_normal((B, N, d)) * 3).astype(dt)
    lab = rng.integers(0, K - 5, (B, N)).astype(np.int32)  # the last 5 clusters are empty
    C_prev = rng.standard_normal((B, K, d)).astype(np.float32)
    C_out, sums, counts = oracle.update(X, lab, C_prev)
    assert (counts.sum(axis=1) == N).all()
    for b in range(B):
        for k in range(K):
            members = X[b][lab[b] == k].astype(np.float64)
            assert counts[b, k] == len(members)
            if len(members) == 0:
                assert np.array_equal(C_out[b, k].view(np.uint32), C_prev[b, k].view(np.uint32))
                assert (sums[b, k] == 0).all()
            else:
                np.testing.assert_allclose(sums[b, k], members.sum(axis=0), rtol=1e-13, atol=1e-12)
                want = members.mean(axis=0).astype(np.float32)
                # both are correctly rounded means up to one fp32 ulp from the double sum order
                assert np.all(np.abs(C_out[b, k].astype(np.float64) - want) <= np.spacing(np.abs(want)))


def test_update_minimises_the_cost_for_fixed_labels():
    rng = np.random.default_rng(8)
    w = synth.small(B=1, N=600, d=8, K=6, dtype="f32", sigma=1.0)
    X = synth.points(w)
    lab = rng.integers(0, w.K, (1, w.N)).astype(np.int32)
    C_out, _, _ = oracle.update(X, lab, np.zeros((1, w.K, w.d), np.float32))
    X64 = X[0].astype(np.float64)

    def J(C):
        return float(((X64 - C[lab[0]]) ** 2).sum())

    base = J(C_out[0].astype(np.float64))
    for _ in range(50):
        delta = rng.standard_normal(C_out[0].shape) * 10.0 ** rng.uniform(-4, 0)
        assert J(C_out[0].astype(np.float64) + delta) >= base - 1e-9 * base


# ---- whole iterations ---------------------------------------------------------

def _frac_to_f32(s):
    f = Fraction(s)
    return np.float32(float(f))


@pytest.mark.parametrize("dt", [np.float32, np.float16])
def test_hand_worked_examples(dt):
    spec = json.load(open(GOLDEN))
    for ex in spec["examples"]:
        X = np.array(ex["X"], dtype=np.float64)[None].astype(dt)
        C = np.array(ex["C0"], dtype=np.float32)[None]
        for t, it in enumerate(ex["iterations"]):
            lab, d1, _ = oracle.assign(X, C)
            assert lab[0].tolist() == it["labels"], (ex["name"], t)
            Jw = float(Fraction(it["J"]))
            tol = 1e-6 if dt == np.float32 else 2e-3
            assert abs(d1.sum() - Jw) <= tol * max(1.0, Jw), (ex["name"], t, d1.sum(), Jw)
            C, _, _ = oracle.update(X, lab, C)
            want = np.array([[_frac_to_f32(v) for v in row] for row in it["C_next"]], dtype=np.float32)
            assert np.array_equal(C[0], want), (ex["name"], t, C[0], want)
        # the full loop reproduces the same trajectory
        lab, C_end, obj = oracle.lloyd(X, np.array(ex["C0"], dtype=np.float32)[None], len(ex["iterations"]))
        assert lab[0].tolist() == ex["iterations"][-1]["labels"]
        assert np.array_equal(C_end, C)


@pytest.mark.parametrize("dt", [np.float32, np.float16])
def test_convergence_stopping_follows_the_hand_worked_shifts(dt):
    spec = json.load(open(GOLDEN))
    examples = {ex["name"]: ex for ex in spec["examples"]}
    for case in spec["stopping"]["cases"]:
        ex = examples[case["example"]]
        X = np.array(ex["X"], dtype=np.float64)[None].astype(dt)
        C0 = np.array(ex["C0"], dtype=np.float32)[None]
        want = [float(Fraction(v)) for v in case["shifts"]]
        for run in case["runs"]:
            tol = float(Fraction(run["tol"]))
            t, lab, C, obj, shift = oracle.lloyd_tol(X, C0, run["max_iters"], tol)
            assert t == run["iters_run"], (case["example"], run, t)
            # the shifts of the iterations run (centroids are fp32: 20/3 is rounded)
            for i in range(t):
                assert abs(shift[i, 0] - want[i]) <= 1e-6 * max(1.0, want[i]), (case["example"], i, shift[i, 0])
            # and the state is that of the plain loop run for the same number of iterations
            lab_p, C_p, obj_p = oracle.lloyd(X, C0, t)
            assert np.array_equal(lab, lab_p) and np.array_equal(C, C_p) and np.array_equal(obj, obj_p)


def test_convergence_stopping_waits_for_every_batch_and_respects_the_cap():
    # two batches: the first settles after 2 iterations (the 2-d square), the second after 3
    # (the 1-d clusters, embedded in 2-d with a zero coordinate); the loop stops for both at 3
    Xa = np.array([[0, 0], [0, 2], [4, 0], [4, 2]], dtype=np.float32)
    Xb = np.array([[0, 0], [1, 0], [9, 0], [10, 0]], dtype=np.float32)
    X = np.stack([Xa, Xb])
    C0 = np.stack([Xa[[0, 1]], Xb[[0, 1]]]).astype(np.float32)
    t, lab, C, obj, shift = oracle.lloyd_tol(X, C0, 10, 0.0)
    assert t == 3
    assert shift[1, 0] == 0.0 and shift[1, 1] > 0.0 and (shift[2] == 0.0).all()
    t, *_ = oracle.lloyd_tol(X, C0, 2, 0.0)
    assert t == 2
    # a negative tolerance is never met: the loop runs to the cap, like the plain loop
    t, lab, C, obj, shift = oracle.lloyd_tol(X, C0, 4, -1.0)
    lab_p, C_p, obj_p = oracle.lloyd(X, C0, 4)
    assert t == 4 and np.array_equal(lab, lab_p) and np.array_equal(C, C_p)


def test_lloyd_reaches_the_global_optimum_on_separable_data():
    # three tight, far-apart groups; from one seed point per group, Lloyd's
    # fixed point is the optimal 3-partition, which enumeration finds exactly.
    X = np.array([[0, 0], [1, 0], [0, 1], [20, 20], [21, 20], [40, 0], [41, 1]], dtype=np.float32)
    C0 = X[[0, 3, 5]].astype(np.float32)
    lab, C, obj = oracle.lloyd(X[None], C0[None], 6)
    best = None
    for part in itertools.product(range(3), repeat=len(X)):
        cost = Fraction(0)
        for k in range(3):
            pts = [X[i] for i in range(len(X)) if part[i] == k]
            if not pts:
                continue
            mean = [sum(Fraction(float(p[j])) for p in pts) / len(pts) for j in range(2)]
            cost += sum((Fraction(float(p[j])) - mean[j]) ** 2 for p in pts for j in range(2))
        best = cost if best is None or cost < best else best
    final = float(oracle.cost(X[None], C.astype(np.float64), lab)[0])
    # C is rounded to fp32 between iterations, so equality holds to fp32 precision
    assert abs(final - float(best)) <= 1e-5 * float(best)
    assert abs(obj[-1, 0] - float(best)) <= 1e-5 * float(best)


@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_objective_never_increases_beyond_centroid_rounding(dtype):
    # J_{t+1} <= J_t + R_{t+1}: the exact mean never increases the cost for
    # fixed labels and reassignment never increases it for fixed centroids;
    # R bounds what rounding the centroid (to fp32, then to X's dtype) can add.
    w = synth.small(B=2, N=3000, d=16, K=25, dtype=dtype, ncomp=20, sigma=0.5, seed=99)
    X = synth.points(w)
    C = synth.init_centroids(w, X)
    code = oracle.F16 if dtype == "f16" else oracle.F32
    prev_J = None
    for t in range(8):
        lab, d1, _ = oracle.assign(X, C)
        J = d1.sum(axis=1)
        if prev_J is not None:
            assert (J <= prev_J + R + 1e-12 * prev_J).all(), (t, J, prev_J, R)
        C_new, sums, counts = oracle.update(X, lab, C)
        mu = np.where(counts[..., None] > 0, sums / np.maximum(counts, 1)[..., None], 0.0)
        chat = oracle.round_centroids(C_new, code)
        # exact cost of the old labels at the rounded new centroids minus at the exact means
        R = np.array([((chat[b] - mu[b]) ** 2).sum(axis=1) @ counts[b] for b in range(w.B)])
        # and the old labels at the exact means cost no more than at the old rounded centroids
        J_mu = oracle.cost(X, mu, lab)
        assert (J_mu <= J * (1 + 1e-12)).all()
        prev_J, C = J, C_new
