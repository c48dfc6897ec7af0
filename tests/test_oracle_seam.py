"""Pins of the oracle's overlap projection and seam discrepancy."""
import os

import numpy as np
import pytest

import synth
from oracle import schedule, seam
from oracle.ddim import ddim_run

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiling_geometry.txt")


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            k, v = line.split()
            out[k] = int(v)
    return out


def test_tiling_geometry_matches_the_page():
    g = _golden()
    assert g["overlap_beads"] * g["bin_kb"] == g["overlap_kb"]
    assert seam.unique_beads(g["chr22_tiles"], g["beads_per_tile"], g["overlap_beads"]) == \
        g["chr22_unique_beads"]
    assert seam.n_seams(g["chr22_tiles"]) == g["chr22_seams"]
    assert synth.chain_beads(g["chr22_tiles"], g["overlap_beads"]) == g["chr22_unique_beads"]
    # the projection writes one o x o block per seam side: 144 of 4096 entries
    assert g["overlap_beads"] ** 2 == 144


def _brute_project(X, o):
    Y = X.copy()
    C, T, B, n, _ = X.shape
    for c in range(C):
        for k in range(T - 1):
            for b in range(B):
                for i in range(o):
                    for j in range(o):
                        m = 0.5 * (X[c, k, b, n - o + i, n - o + j] + X[c, k + 1, b, i, j])
                        Y[c, k, b, n - o + i, n - o + j] = m
                        Y[c, k + 1, b, i, j] = m
    return Y


@pytest.mark.parametrize("o", [1, 5, 12, 32])
def test_projection_brute_force(o):
    X = np.random.default_rng(o).standard_normal((2, 3, 2, 64, 64))
    np.testing.assert_array_equal(seam.seam_project(X, o), _brute_project(X, o))


def test_projection_properties():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((2, 5, 3, 64, 64))
    X = X + np.swapaxes(X, -1, -2)
    P = seam.seam_project(X)
    np.testing.assert_array_equal(seam.seam_project(P), P)                         # idempotent
    np.testing.assert_array_equal(P[:, :-1, :, 52:, 52:], P[:, 1:, :, :12, :12])   # agree
    np.testing.assert_array_equal(P, np.swapaxes(P, -1, -2))                       # symmetric
    mask = np.ones((5, 64, 64), dtype=bool)
    mask[:-1, 52:, 52:] = False
    mask[1:, :12, :12] = False
    np.testing.assert_array_equal(P.swapaxes(1, 2)[:, :, mask], X.swapaxes(1, 2)[:, :, mask])  # rest unchanged
    perm = rng.permutation(3)
    np.testing.assert_array_equal(seam.seam_project(X[:, :, perm]), P[:, :, perm])  # per sample
    # a single tile has nothing to project
    np.testing.assert_array_equal(seam.seam_project(X[:, :1]), X[:, :1])


def _brute_discrepancy(X, o):
    C, T, B, n, _ = X.shape
    out = np.zeros((C, T - 1))
    for c in range(C):
        for k in range(T - 1):
            tot = 0.0
            for i in range(o):
                for j in range(o):
                    a = sum(X[c, k, b, n - o + i, n - o + j] for b in range(B)) / B
                    bb = sum(X[c, k + 1, b, i, j] for b in range(B)) / B
                    tot += abs(a - bb)
            out[c, k] = tot / (o * o)
    return out


@pytest.mark.parametrize("o", [3, 12])
def test_discrepancy_brute_force_and_shards(o):
    X = np.random.default_rng(2).standard_normal((2, 3, 4, 64, 64))
    ref = _brute_discrepancy(X, o)
    np.testing.assert_allclose(seam.seam_discrepancy(X, o), ref, rtol=1e-13)
    # split the samples into shards: summed overlap differences give the same
    sums = seam.overlap_difference_sums(X[:, :, :1], o) + seam.overlap_difference_sums(X[:, :, 1:], o)
    np.testing.assert_allclose(seam.discrepancy_from_sums(sums, 4), ref, rtol=1e-13)
    assert np.all(seam.seam_discrepancy(seam.seam_project(X, o), o) == 0.0)


def test_unsynchronised_discrepancy_statistics():
    # Without projection the final overlap difference of a seam is
    # -c0 (eps~_k - eps~_{k+1}) with eps~ = (1+w) s_c z_c - w s_u z_u, so the
    # per-sample mean is N(0, 2 s_eff^2 / B) per independent entry and
    # E|.| = c0 s_eff sqrt(2/B) sqrt(2/pi).
    S, T, B, w, s_c, s_u = 2, 6, 400, 1.0, 0.1, 0.3
    s = schedule.Schedule(S=S)
    x0 = synth.chain_x0(3, 1, T).astype(np.float64)
    out = ddim_run(x0, s, w, s_c, s_u, 5, np.arange(B), B, sync_every=0)
    d = seam.seam_discrepancy(out)
    c0 = np.sqrt(1 - s.ab_t[0]) / np.sqrt(s.ab_t[0])
    s_eff = np.hypot((1 + w) * s_c, w * s_u)
    expect = c0 * s_eff * np.sqrt(2.0 / B) * np.sqrt(2.0 / np.pi)
    # 78 independent entries per seam, 5 seams: relative spread ~ 0.75/sqrt(390)
    assert abs(d.mean() / expect - 1.0) < 0.15, (d.mean(), expect)
    # and projecting after the last step drives it to zero
    out_sync = ddim_run(x0, s, w, s_c, s_u, 5, np.arange(B), B, sync_every=1)
    assert np.all(seam.seam_discrepancy(out_sync) == 0.0)
