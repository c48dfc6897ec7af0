"""GPU parity of SMACOF coordinate refinement against the float64 oracle, on
noisy point-cloud maps started from perturbed ground-truth coordinates."""
import numpy as np
import pytest

import synth
from oracle import refine as oref
from tests.gpu_util import dev, host, needs_gpu, torch

pytestmark = [pytest.mark.gpu, needs_gpu]

TOL_REFINE = 1e-4    # coordinates, normwise per map; stress, relative


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


def _start(seed, count, jitter=0.05):
    """Noisy maps of the point-cloud workload and a start near their points."""
    maps, pts, sig = synth.cloud_block(seed, 0)
    g = np.random.default_rng([seed, 0x5EED])
    X0 = pts + jitter * sig[:, None, None] * g.standard_normal(pts.shape)
    return maps[:count], X0[:count].astype(np.float32)


def _refine(tdm, maps, X0, iterations, want_stress=True):
    n = maps.shape[0]
    coords = dev(X0).reshape(-1).clone()
    stress = torch.empty(max(n, 1), device="cuda") if want_stress else None
    tdm.refine_smacof(dev(maps).reshape(-1), n, coords, iterations, stress)
    torch.cuda.synchronize()
    return host(coords).reshape(n, 64, 3), (host(stress)[:n] if want_stress else None)


def _normwise(X, Y):
    return np.abs(X - Y).max(axis=(1, 2)) / np.abs(Y).max(axis=(1, 2))


@pytest.mark.parametrize("count,iterations", [(1, 5), (131, 30), (600, 12)])
def test_refine_matches_oracle(tdm, count, iterations):
    maps, X0 = _start(1, count)
    X, s = _refine(tdm, maps, X0, iterations)
    Xo, so = oref.smacof(X0.astype(np.float64), maps.astype(np.float64), iterations)
    e = _normwise(X, Xo)
    assert e.max() <= TOL_REFINE, f"coordinates: {e.max():.3e} at map {int(np.argmax(e))}"
    es = np.abs(s - so) / so
    assert es.max() <= TOL_REFINE, f"stress: {es.max():.3e}"
    # the reported stress is the stress of the returned coordinates
    np.testing.assert_allclose(s, oref.stress(X, maps.astype(np.float64)), rtol=TOL_REFINE)


def test_refine_reduces_stress(tdm):
    maps, X0 = _start(2, 200, jitter=0.3)
    s0 = oref.stress(X0.astype(np.float64), maps.astype(np.float64))
    _, s = _refine(tdm, maps, X0, 25)
    assert np.all(s < s0)


def test_zero_iterations_keep_coordinates(tdm):
    maps, X0 = _start(3, 9)
    X, s = _refine(tdm, maps, X0, 0)
    np.testing.assert_array_equal(X, X0.astype(np.float64))
    np.testing.assert_allclose(s, oref.stress(X0.astype(np.float64), maps.astype(np.float64)), rtol=TOL_REFINE)


def test_exact_distances_are_a_fixed_point(tdm):
    pts = synth.random_points(4, 40, scale=3.0)
    D = synth.exact_distance_maps(pts).astype(np.float32)
    X0 = (pts - pts.mean(axis=1, keepdims=True)).astype(np.float32)
    X, s = _refine(tdm, D, X0, 20)
    assert _normwise(X, X0.astype(np.float64)).max() <= TOL_REFINE
    assert np.all(s <= 1e-8 * (D.astype(np.float64) ** 2).sum(axis=(1, 2)))


def test_coincident_beads_and_asymmetric_maps(tdm):
    # two beads start on the same point (their pair term is left out), and the
    # maps are not symmetric (both sides symmetrise them first)
    maps, X0 = _start(5, 12)
    X0[:, 7] = X0[:, 3]
    g = np.random.default_rng(11)
    maps = (maps * (1.0 + 0.02 * g.standard_normal(maps.shape))).astype(np.float32)
    X, s = _refine(tdm, maps, X0, 10)
    Xo, so = oref.smacof(X0.astype(np.float64), maps.astype(np.float64), 10)
    assert _normwise(X, Xo).max() <= TOL_REFINE
    assert (np.abs(s - so) / so).max() <= TOL_REFINE


def test_no_maps_and_no_stress_output(tdm):
    maps, X0 = _start(6, 4)
    tdm.refine_smacof(dev(maps).reshape(-1), 0, dev(X0).reshape(-1), 3)
    X, s = _refine(tdm, maps, X0, 6, want_stress=False)
    Xo, _ = oref.smacof(X0.astype(np.float64), maps.astype(np.float64), 6)
    assert s is None and _normwise(X, Xo).max() <= TOL_REFINE


def test_refine_full_size_sampled(tdm):
    # the 32,000 final maps of the 32-tile x 1000-sample chain workload: a sample
    # of maps against the oracle, stress decrease on all of them
    n = 32000
    blk = synth.CLOUD_BLOCK
    maps = synth.cloud_maps(0, 0, n)
    X0 = np.empty((n, 64, 3), dtype=np.float32)
    g = np.random.default_rng([0, 0x5EED])
    for b0 in range(0, n, blk):
        _, pts, sig = synth.cloud_block(0, b0 // blk)
        k = min(blk, n - b0)
        X0[b0:b0 + k] = (pts[:k] + 0.05 * sig[:k, None, None] * g.standard_normal((k, 64, 3)))
    X, s = _refine(tdm, maps, X0, 20)
    idx = np.random.default_rng(9).choice(n, 48, replace=False)
    idx = np.unique(np.concatenate([idx, [0, n - 1]]))
    Xo, so = oref.smacof(X0[idx].astype(np.float64), maps[idx].astype(np.float64), 20)
    assert _normwise(X[idx], Xo).max() <= TOL_REFINE
    assert (np.abs(s[idx] - so) / so).max() <= TOL_REFINE
    s0 = np.concatenate([oref.stress(X0[i:i + 2000].astype(np.float64), maps[i:i + 2000].astype(np.float64))
                         for i in range(0, n, 2000)])
    assert np.all(s < s0)
