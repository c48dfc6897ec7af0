"""Pins of the oracle's SMACOF refinement."""
import numpy as np

import synth
from oracle import mds, refine


def test_guttman_step_is_a_gradient_step():
    # for centred X the Guttman transform equals X - grad(sigma) / (2n),
    # checked against a central finite-difference gradient of the stress
    g = np.random.default_rng(0)
    pts = synth.random_points(1, 1, n=16)[0]
    D = synth.exact_distance_maps(pts) * (1 + 0.05 * g.standard_normal((16, 16)))
    D = 0.5 * (D + D.T)
    np.fill_diagonal(D, 0.0)
    X = pts + 0.3 * g.standard_normal(pts.shape)
    X -= X.mean(axis=0)
    grad = np.zeros_like(X)
    h = 1e-6
    for i in range(16):
        for a in range(3):
            Xp, Xm = X.copy(), X.copy()
            Xp[i, a] += h
            Xm[i, a] -= h
            grad[i, a] = (refine.stress(Xp, D) - refine.stress(Xm, D)) / (2 * h)
    np.testing.assert_allclose(refine.guttman_transform(X, D), X - grad / (2 * 16), atol=1e-6)


def test_stress_never_increases():
    maps = synth.cloud_maps(0, 0, 4).astype(np.float64)
    X0 = synth.random_points(2, 4) * 5.0
    prev = refine.stress(X0, maps)
    X = X0
    for _ in range(20):
        X = refine.guttman_transform(X, 0.5 * (maps + np.swapaxes(maps, 1, 2)))
        cur = refine.stress(X, maps)
        assert np.all(cur <= prev * (1 + 1e-12))
        prev = cur


def test_exact_distances_are_a_fixed_point():
    pts = synth.random_points(3, 5, scale=4.0)
    D = synth.exact_distance_maps(pts)
    X0, _ = mds.classical_mds(D)
    X, s = refine.smacof(X0, D, 10)
    np.testing.assert_allclose(X, X0 - X0.mean(axis=1, keepdims=True), atol=1e-9)
    assert np.all(s < 1e-15 * (D ** 2).sum(axis=(1, 2)))


def test_refinement_reduces_stress_of_the_initialisation():
    # with noisy maps classical MDS is not the stress minimiser
    maps = synth.cloud_maps(0, 0, 8).astype(np.float64)
    X0, _ = mds.classical_mds(maps)
    s0 = refine.stress(X0, maps)
    _, s = refine.smacof(X0, maps, 30)
    assert np.all(s < s0)
