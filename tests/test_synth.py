"""The seeded input generator: known-answer Philox vectors, chunk regeneration, mixture statistics."""
import numpy as np
import pytest

import synth


def test_philox4x32_10_known_answers():
    # Known-answer vectors published with the Random123 library (Salmon et al., SC'11).
    assert synth.philox4x32_10([0, 0, 0, 0], [0, 0]) == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]
    assert synth.philox4x32_10([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2) == [0x408F276D, 0x41C83B0E, 0xA20BC7C6,
                                                                       0x6D5451FD]
    assert synth.philox4x32_10([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0]) == [
        0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_any_row_range_regenerates_identically(dtype):
    w = synth.small(B=3, N=2000, d=20, K=7, dtype=dtype)
    full = synth.points(w)
    part = synth.points(w, row0=777, nrows=555)
    assert np.array_equal(full[:, 777:777 + 555].view(np.uint8), part.view(np.uint8))
    assert np.array_equal(synth.points(w).view(np.uint8), full.view(np.uint8))  # deterministic


def test_normals_have_unit_moments():
    z = synth.normals(1234, 3, 0, 0, 50000, 8).ravel()
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01


def test_mixture_components_and_spread():
    w = synth.small(B=1, N=40000, d=16, K=5, dtype="f32", ncomp=5, sigma=0.25, seed=77)
    X, comp = synth.points(w, with_components=True)
    freq = np.bincount(comp[0], minlength=5) / w.N
    assert np.all(np.abs(freq - 0.2) < 0.01)
    for c in range(5):
        pts = X[0][comp[0] == c].astype(np.float64)
        assert abs(pts.std(axis=0).mean() - 0.25) < 0.01


def test_zipf_weights():
    w = synth.small(B=1, N=200000, d=4, K=100, dtype="f16", ncomp=100, zipf=1.2, seed=5)
    _, comp = synth.points(w, with_components=True)
    freq = np.bincount(comp[0], minlength=100) / w.N
    r = np.arange(1, 101, dtype=np.float64)
    want = r ** -1.2 / (r ** -1.2).sum()
    assert np.all(np.abs(freq - want) < 5 * np.sqrt(want / w.N) + 1e-4)


def test_init_indices_are_distinct_and_in_range():
    w = synth.small(B=4, N=500, d=4, K=300)
    idx = synth.init_indices(w)
    for b in range(w.B):
        assert len(set(idx[b].tolist())) == w.K
        assert idx[b].min() >= 0 and idx[b].max() < w.N
    assert not np.array_equal(idx[0], idx[1])
