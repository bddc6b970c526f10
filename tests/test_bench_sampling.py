"""The bench's CPU leg: the oracle runs on a bounded sample of the workload and is scaled to the whole
iteration, whether the sample is whole problems or, when one problem alone exceeds the time budget, the
first points of one problem (CPU only)."""
import importlib.util
import os

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_whole_problems_when_they_fit(bench):
    w = synth.small(B=6, N=3000, d=32, K=20, dtype="f16", seed=5)
    nb, rows = bench.oracle_sample(w, 60.0)
    assert rows == w.N and nb == w.B
    assert bench.sample_scale(w, nb, rows) == 1.0
    assert "the whole iteration" in bench.cpu_sample_text(w, nb, rows, 1.0)


def test_row_sample_of_one_problem_when_one_is_too_long(bench):
    # a budget far below one problem's time: the first rows of problem 0, scaled by B and N / rows
    w = synth.small(B=3, N=200000, d=64, K=500, dtype="f16", seed=6)
    nb, rows = bench.oracle_sample(w, 1e-3)
    assert nb == 1 and 2048 <= rows < w.N
    assert bench.sample_scale(w, nb, rows) == pytest.approx(w.B * w.N / rows)
    text = bench.cpu_sample_text(w, nb, rows, 1.0)
    assert f"the first {rows} of the {w.N} points of problem 0" in text


def test_parity_report_on_a_row_sample(bench):
    import numpy as np
    import oracle
    w = synth.small(B=2, N=4000, d=32, K=30, dtype="f16", seed=7)
    X = synth.points(w)
    C = synth.init_centroids(w, X)
    lab, _, _ = oracle.assign(X, C)
    dt, rep = bench.parity_report(w, X, C, lab.astype(np.int32), 1, 1500)
    assert rep["checked_points"] == 1500
    assert rep["label_mismatches_at_clear_points"] == 0 and rep["label_mismatches_at_near_ties"] == 0
    wrong = lab.copy()
    wrong[0, :1500] = (wrong[0, :1500] + 1) % w.K  # every sampled label off by one
    _, rep = bench.parity_report(w, X, C, wrong.astype(np.int32), 1, 1500)
    assert rep["label_mismatches_at_clear_points"] + rep["label_mismatches_at_near_ties"] == 1500
