"""Pins of the oracle's classical MDS and distance reconstruction."""
import numpy as np
import pytest

import synth
from oracle import mds


def test_exact_euclidean_distances_are_reproduced():
    pts = synth.random_points(3, 6, scale=4.0)
    D = synth.exact_distance_maps(pts)
    X, lam = mds.classical_mds(D)
    R = mds.pairwise_distances(X)
    assert np.abs(R - D).max() / np.abs(D).max() < 1e-9
    # rank 3: the remaining eigenvalues vanish
    assert np.all(np.abs(lam[:, 3:]) < 1e-9 * lam[:, :1])


def test_eigenvalues_equal_the_scatter_matrix_spectrum():
    # B = Xc Xc^T for centred coordinates Xc, so its nonzero eigenvalues are
    # those of the 3 x 3 scatter matrix Xc^T Xc
    pts = synth.random_points(4, 5)
    D = synth.exact_distance_maps(pts)
    _, lam = mds.classical_mds(D)
    for p, l in zip(pts, lam):
        xc = p - p.mean(axis=0)
        ref = np.sort(np.linalg.eigvalsh(xc.T @ xc))[::-1]
        np.testing.assert_allclose(l[:3], ref, rtol=1e-10)


def test_jacobi_agrees_with_library_eigh():
    maps = synth.cloud_maps(0, 0, 4).astype(np.float64)
    B = mds.double_center(maps * maps)
    lam, V, sweeps = mds.jacobi_eigh(B)
    order = np.argsort(-lam, axis=-1)
    lam = np.take_along_axis(lam, order, -1)
    V = np.take_along_axis(V, order[:, None, :], -1)
    ref_l, ref_v = np.linalg.eigh(B)
    ref_l, ref_v = ref_l[:, ::-1], ref_v[:, :, ::-1]
    np.testing.assert_allclose(lam, ref_l, rtol=0, atol=1e-10 * np.abs(ref_l).max())
    for k in range(3):
        dots = np.abs(np.einsum("ni,ni->n", V[:, :, k], ref_v[:, :, k]))
        np.testing.assert_allclose(dots, 1.0, atol=1e-9)
    # B = V diag(lam) V^T, V orthogonal
    np.testing.assert_allclose(V @ (lam[:, :, None] * np.swapaxes(V, 1, 2)), B, atol=1e-9 * np.abs(B).max())
    np.testing.assert_allclose(np.swapaxes(V, 1, 2) @ V, np.broadcast_to(np.eye(64), V.shape), atol=1e-12)
    assert sweeps < 30


def test_permutation_equivariance_and_symmetrisation():
    D = synth.cloud_maps(1, 5, 2).astype(np.float64)
    perm = np.random.default_rng(0).permutation(64)
    X, lam = mds.classical_mds(D)
    Xp, lamp = mds.classical_mds(D[:, perm][:, :, perm])
    np.testing.assert_allclose(lamp, lam, rtol=1e-9, atol=1e-9 * lam.max())
    np.testing.assert_allclose(mds.pairwise_distances(Xp), mds.pairwise_distances(X)[:, perm][:, :, perm],
                               atol=1e-8 * D.max())
    # an asymmetric input is read through its symmetric part
    A = D + np.random.default_rng(1).standard_normal(D.shape) * 0.01
    Xa, la = mds.classical_mds(A)
    Xs, ls = mds.classical_mds(0.5 * (A + np.swapaxes(A, 1, 2)))
    np.testing.assert_allclose(la, ls, rtol=1e-12, atol=1e-9)


def test_negative_eigenvalues_are_clamped():
    # a non-Euclidean "distance" map: coordinates built only from the
    # non-negative part of the top three eigenvalues
    rng = np.random.default_rng(2)
    D = np.abs(rng.standard_normal((1, 64, 64)))
    D = D + D.transpose(0, 2, 1)
    np.fill_diagonal(D[0], 0.0)
    X, lam = mds.classical_mds(D)
    for k in range(3):
        np.testing.assert_allclose(np.linalg.norm(X[0, :, k]) ** 2, max(lam[0, k], 0.0), rtol=1e-9, atol=1e-12)


def test_pairwise_distances_brute_force():
    X = np.random.default_rng(3).standard_normal((2, 7, 3))
    R = mds.pairwise_distances(X)
    for n in range(2):
        for i in range(7):
            for j in range(7):
                assert abs(R[n, i, j] - np.sqrt(sum((X[n, i, d] - X[n, j, d]) ** 2 for d in range(3)))) < 1e-15
    assert np.all(np.diagonal(R, axis1=1, axis2=2) == 0.0)


@pytest.mark.parametrize("mistake", ["no_half", "single_center", "no_square"])
def test_pins_catch_planted_mistakes(mistake, monkeypatch):
    # plant a plausible mistake in the oracle and check the exact-distance pin fails
    pts = synth.random_points(6, 2)
    D = synth.exact_distance_maps(pts)
    orig = mds.double_center
    if mistake == "no_half":
        monkeypatch.setattr(mds, "double_center", lambda D2: -(2.0 * orig(D2)))
    elif mistake == "single_center":
        def one_side(D2):
            n = D2.shape[-1]
            J = np.eye(n) - np.ones((n, n)) / n
            return -0.5 * (J @ D2)
        monkeypatch.setattr(mds, "double_center", one_side)
    else:
        monkeypatch.setattr(mds, "double_center", lambda D2: orig(np.sqrt(D2)))
    X, _ = mds.classical_mds(D)
    err = np.abs(mds.pairwise_distances(X) - D).max() / D.max()
    assert err > 1e-3
