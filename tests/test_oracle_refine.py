"""Pins of the oracle's SMACOF refinement."""
import numpy as np
import pytest

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


def test_transposed_maps_give_the_same_refinement():
    # the map is symmetrised first, so D and D^T refine alike
    g = np.random.default_rng(4)
    pts = synth.random_points(7, 2, n=20)
    D = synth.exact_distance_maps(pts) * (1 + 0.05 * g.standard_normal((2, 20, 20)))
    X0 = pts + 0.2 * g.standard_normal(pts.shape)
    Xa, sa = refine.smacof(X0, D, 8)
    Xb, sb = refine.smacof(X0, np.swapaxes(D, 1, 2), 8)
    np.testing.assert_allclose(Xa, Xb, atol=1e-12)
    np.testing.assert_allclose(sa, sb, rtol=1e-12)


_PINS = [test_guttman_step_is_a_gradient_step, test_stress_never_increases, test_exact_distances_are_a_fixed_point,
         test_transposed_maps_give_the_same_refinement]


@pytest.mark.parametrize("mistake", ["n_minus_1", "sign", "no_diagonal", "squared_weights", "no_symmetrise"])
def test_pins_catch_planted_mistakes(mistake, monkeypatch):
    # plant a plausible mistake in the oracle; at least one pin must fail
    orig_gt = refine.guttman_transform

    def bad_gt(X, D):
        X = np.asarray(X, dtype=np.float64)
        n = X.shape[-2]
        d = refine.pairwise(X)
        safe = np.where(d > 0.0, d, 1.0)
        w = D / safe if mistake != "squared_weights" else (D / safe) ** 2
        Bm = np.where(d > 0.0, -w if mistake != "sign" else w, 0.0)
        idx = np.arange(n)
        Bm[..., idx, idx] = 0.0
        if mistake != "no_diagonal":
            Bm[..., idx, idx] = -Bm.sum(axis=-1)
        return Bm @ X / (n - 1 if mistake == "n_minus_1" else n)

    def bad_smacof(X0, D, iterations):
        X = np.asarray(X0, dtype=np.float64)
        for _ in range(iterations):
            X = orig_gt(X, np.asarray(D, dtype=np.float64))
        return X, refine.stress(X, D)

    if mistake == "no_symmetrise":
        monkeypatch.setattr(refine, "smacof", bad_smacof)
    else:
        monkeypatch.setattr(refine, "guttman_transform", bad_gt)
    failed = 0
    for pin in _PINS:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, f"no pin caught {mistake}"
