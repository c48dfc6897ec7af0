"""GPU parity of coordinate recovery (classical MDS) and distance
reconstruction against the float64 oracle.  Coordinates are unique only up to
rotation and reflection, so they are compared through the distance maps they
rebuild and after an orthogonal Procrustes fit."""
import numpy as np
import pytest

import synth
from oracle import mds as omds
from tests.gpu_util import TOL_RECOVER, dev, host, needs_gpu, normwise, torch

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


def _recover(tdm, maps):
    n = maps.shape[0]
    coords = torch.empty(n * 192, device="cuda")
    eig = torch.empty(n * 3, device="cuda")
    tdm.mds_recover(dev(maps).reshape(-1), n, coords, eig)
    flags = tdm.ctx_sync()
    return host(coords).reshape(n, 64, 3), host(eig).reshape(n, 3), flags


def _procrustes_err(X, Y):
    """min over orthogonal Q of ||X Q - Y|| / ||Y|| (reflections allowed)."""
    Xc, Yc = X - X.mean(0), Y - Y.mean(0)
    u, _, vt = np.linalg.svd(Xc.T @ Yc)
    return np.linalg.norm(Xc @ (u @ vt) - Yc) / max(np.linalg.norm(Yc), 1e-30)


def _check(tdm, maps, what):
    X, lam, flags = _recover(tdm, maps)
    assert flags == 0, f"{what}: MDS flagged non-convergence"
    Xo, lo = omds.classical_mds(maps.astype(np.float64))
    Ro = omds.pairwise_distances(Xo)
    e = normwise(omds.pairwise_distances(X), Ro)
    assert e.max() <= TOL_RECOVER, f"{what}: rebuilt distances {e.max():.3e}"
    el = np.abs(lam - lo[:, :3]).max(axis=1) / np.abs(lo[:, 0])
    assert el.max() <= TOL_RECOVER, f"{what}: eigenvalues {el.max():.3e}"
    # coordinates up to an orthogonal map, where the top three are well separated
    gap = (lo[:, 2] - lo[:, 3]) / lo[:, 0]
    for k in np.nonzero(gap > 1e-3)[0]:
        assert _procrustes_err(X[k], Xo[k]) <= 1e-3, f"{what}: coordinates of map {k}"
    return X, lam


def test_mds_on_noisy_point_clouds(tdm):
    maps = synth.cloud_maps(0, 0, 96)
    _check(tdm, maps, "noisy clouds")


def test_mds_recovers_exact_distances(tdm):
    pts = synth.random_points(5, 64, scale=3.0)
    D = synth.exact_distance_maps(pts).astype(np.float32)
    X, _ = _check(tdm, D, "exact clouds")
    R = omds.pairwise_distances(X)
    assert normwise(R, D).max() <= 1e-5


def test_mds_edge_maps(tdm):
    # an all-zero map, a tiny-scale map, a huge-scale map, an asymmetric map
    pts = synth.random_points(8, 3)
    D = synth.exact_distance_maps(pts)
    maps = np.stack([np.zeros((64, 64)), D[0] * 1e-6, D[1] * 1e5,
                     D[2] + np.random.default_rng(0).standard_normal((64, 64)) * 0.01]).astype(np.float32)
    X, lam, flags = _recover(tdm, maps)
    assert np.all(np.isfinite(X)) and np.all(np.isfinite(lam))
    assert np.all(X[0] == 0) and np.all(lam[0] == 0)
    Xo, lo = omds.classical_mds(maps[1:].astype(np.float64))
    e = normwise(omds.pairwise_distances(X[1:]), omds.pairwise_distances(Xo))
    assert e.max() <= TOL_RECOVER


def test_pairwise_dist_matches_oracle(tdm):
    X = synth.random_points(9, 50, scale=4.0).astype(np.float32)
    out = torch.empty(50 * 4096, device="cuda")
    tdm.pairwise_dist(dev(X).reshape(-1), 50, out)
    g = host(out).reshape(50, 64, 64)
    ref = omds.pairwise_distances(X.astype(np.float64))
    assert normwise(g, ref).max() <= 1e-6
    np.testing.assert_array_equal(g, np.swapaxes(g, 1, 2))
    assert np.all(np.diagonal(g, axis1=1, axis2=2) == 0)


def test_recovery_of_sampler_output(tdm):
    # the whole pipeline on the small tiled chain: GPU sampler -> GPU MDS ->
    # GPU reconstruction against oracle sampler -> oracle MDS -> oracle
    # reconstruction, each side from the same synthetic x0
    from oracle import schedule as osched
    from oracle.ddim import ddim_run as o_run
    wl = synth.WORKLOADS["chain4_b8_s50"]
    t = tdm.Tiling(C=1, T=4, B=8)
    sch = tdm.Schedule(50)
    x0 = synth.chain_x0(wl.seed, 1, 4)
    n = t.n_maps
    maps = torch.empty(n * 4096, device="cuda")
    coords = torch.empty(n * 192, device="cuda")
    rec = torch.empty(n * 4096, device="cuda")
    tdm.ddim_run(sch, maps, dev(x0), 0.0, 0.1, 0.3, wl.seed, t)
    tdm.mds_recover(maps, n, coords)
    tdm.pairwise_dist(coords, n, rec)
    assert tdm.ctx_sync() == 0
    ref = o_run(x0, osched.Schedule(S=50), 0.0, 0.1, 0.3, wl.seed, np.arange(8), 8).reshape(-1, 64, 64)
    Xo, _ = omds.classical_mds(ref)
    e = normwise(host(rec).reshape(-1, 64, 64), omds.pairwise_distances(Xo))
    assert e.max() <= TOL_RECOVER, e.max()


def test_mds_rank_deficient_maps(tdm):
    # points on a plane (lambda_3 = 0) and on a line (lambda_2 = lambda_3 = 0):
    # the distances rebuild, the null eigenvalues come out ~0, and the
    # eigen-solve converges without a flag
    g = np.random.default_rng(3)
    plane = np.concatenate([g.standard_normal((4, 64, 2)) * 3.0, np.zeros((4, 64, 1))], axis=2)
    line = np.concatenate([g.standard_normal((4, 64, 1)) * 3.0, np.zeros((4, 64, 2))], axis=2)
    rot = np.stack([synth.random_orthogonal(g) for _ in range(8)])
    pts = np.einsum("mij,mnj->mni", rot, np.concatenate([plane, line]))
    D = synth.exact_distance_maps(pts).astype(np.float32)
    X, lam, flags = _recover(tdm, D)
    assert flags == 0 and np.all(np.isfinite(X))
    e = normwise(omds.pairwise_distances(X), D.astype(np.float64))
    assert e.max() <= TOL_RECOVER, e.max()
    assert np.all(np.abs(lam[:4, 2]) <= 1e-5 * lam[:4, 0])
    assert np.all(np.abs(lam[4:, 1:]) <= 1e-5 * lam[4:, :1])


@pytest.mark.parametrize("n", [1, 37, 1000])
def test_fused_reconstruction_equals_the_two_calls(tdm, n):
    # tdm_mds_reconstruct writes the coordinates, eigenvalues and distance
    # maps that tdm_mds_recover followed by tdm_pairwise_dist write, bit for bit
    maps = dev(synth.cloud_maps(2, 0, n)).reshape(-1)
    c1, e1, d1 = (torch.empty(n * k, device="cuda") for k in (192, 3, 4096))
    c2, e2, d2 = (torch.empty(n * k, device="cuda") for k in (192, 3, 4096))
    tdm.mds_recover(maps, n, c1, e1)
    tdm.pairwise_dist(c1, n, d1)
    tdm.mds_reconstruct(maps, n, c2, d2, e2)
    assert tdm.ctx_sync() == 0
    for a, b in ((c1, c2), (e1, e2), (d1, d2)):
        np.testing.assert_array_equal(host(a), host(b))
