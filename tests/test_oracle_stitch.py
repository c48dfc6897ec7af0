"""Pins of the oracle's Kabsch stitching."""
import numpy as np
import pytest

import synth
from oracle import stitch


def test_exact_tiles_rebuild_the_chain():
    # noise-free tiles of one walk under random orthogonal maps (reflections
    # included): the stitched chain is the walk in tile 0's frame, residuals 0
    X, walks, (R, t) = synth.tile_coords(1, 2, 5, 3, noise=0.0)
    chains, res = stitch.stitch(X.astype(np.float64))
    for c in range(2):
        for b in range(3):
            ref = walks[c, b] @ R[c, 0, b].T + t[c, 0, b]
            assert np.abs(chains[c, b] - ref).max() < 1e-4 * np.abs(ref).max()   # float32 inputs
    assert res.max() < 1e-4
    Xd = np.asarray(X, dtype=np.float64)
    # the same from float64 tiles: exact to rounding
    X64 = np.empty_like(Xd)
    for c in range(2):
        for k in range(5):
            for b in range(3):
                X64[c, k, b] = walks[c, b, k * 52:k * 52 + 64] @ R[c, k, b].T + t[c, k, b]
    chains64, res64 = stitch.stitch(X64)
    for c in range(2):
        for b in range(3):
            ref = walks[c, b] @ R[c, 0, b].T + t[c, 0, b]
            np.testing.assert_allclose(chains64[c, b], ref, atol=1e-9)
    assert res64.max() < 1e-10


def test_procrustes_matches_library_kabsch_for_proper_rotations():
    from scipy.spatial.transform import Rotation
    g = np.random.default_rng(3)
    for _ in range(20):
        Q = g.standard_normal((12, 3))
        Rt = synth.random_orthogonal(g, proper=True)
        P = Q @ Rt.T + g.standard_normal(3) + 0.05 * g.standard_normal((12, 3))
        R, t, rmsd = stitch.procrustes(P, Q)
        rot, _ = Rotation.align_vectors(P - P.mean(0), Q - Q.mean(0))
        np.testing.assert_allclose(R, rot.as_matrix(), atol=1e-8)


def test_procrustes_is_optimal():
    from scipy.spatial.transform import Rotation
    g = np.random.default_rng(4)
    P = g.standard_normal((12, 3))
    Q = P @ synth.random_orthogonal(g).T + 0.1 * g.standard_normal((12, 3))
    R, t, rmsd = stitch.procrustes(P, Q)
    assert abs(np.linalg.det(R)) == pytest.approx(1.0)
    for _ in range(200):
        small = Rotation.from_rotvec(g.standard_normal(3) * 0.02).as_matrix()
        for Rc in (small @ R, synth.random_orthogonal(g)):
            tc = P.mean(0) - Rc @ Q.mean(0)
            r = np.sqrt((((Q @ Rc.T + tc) - P) ** 2).sum(1).mean())
            assert r >= rmsd - 1e-12


def test_rigid_changes_of_a_tile_do_not_change_the_chain():
    X, _, _ = synth.tile_coords(5, 1, 4, 2, noise=0.05)
    X = X.astype(np.float64)
    ref, res = stitch.stitch(X)
    g = np.random.default_rng(6)
    Y = X.copy()
    for k in (1, 3):
        Y[0, k, 1] = Y[0, k, 1] @ synth.random_orthogonal(g).T + g.standard_normal(3)
    got, res2 = stitch.stitch(Y)
    np.testing.assert_allclose(got, ref, atol=1e-9)
    np.testing.assert_allclose(res2, res, atol=1e-12)


def test_planted_transpose_fails_the_exact_pin(monkeypatch):
    X, walks, (R, t) = synth.tile_coords(7, 1, 3, 1, noise=0.0)
    orig = stitch.procrustes

    def transposed(P, Q):
        Rr, tt, r = orig(P, Q)
        Rr = Rr.T
        return Rr, P.mean(0) - Rr @ Q.mean(0), r
    monkeypatch.setattr(stitch, "procrustes", transposed)
    chains, _ = stitch.stitch(X.astype(np.float64))
    ref = walks[0, 0] @ R[0, 0, 0].T + t[0, 0, 0]
    assert np.abs(chains[0, 0] - ref).max() > 1e-2
