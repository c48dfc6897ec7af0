"""GPU parity of Kabsch stitching against the float64 oracle."""
import numpy as np
import pytest

import synth
from oracle import stitch as ostitch
from tests.gpu_util import dev, host, needs_gpu, torch

pytestmark = [pytest.mark.gpu, needs_gpu]

# stitched chains, normwise over a chain: float32 polar factors composed over
# up to 39 seams; residuals relative to the oracle's (floor 1e-3 of the
# noise), or both near 0 for noise-free tiles
TOL_CHAIN = 1e-4
TOL_RESID = 1e-3


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


def _run(tdm, X, T, overlap):
    C, _, B = X.shape[:3]
    t = tdm.Tiling(C=C, T=T, B=B, overlap=overlap)
    L = 64 + (T - 1) * (64 - overlap)
    chain = torch.empty(C * B * L * 3, device="cuda")
    res = torch.empty(max(C * B * (T - 1), 1), device="cuda")
    tdm.kabsch_stitch(dev(X).reshape(-1), t, chain, res if T > 1 else None)
    torch.cuda.synchronize()
    return host(chain).reshape(C, B, L, 3), host(res)[:C * B * (T - 1)].reshape(C, B, T - 1)


@pytest.mark.parametrize("C,T,B,o,noise", [(2, 5, 3, 12, 0.05), (1, 32, 8, 12, 0.02), (2, 40, 3, 8, 0.05),
                                           (1, 3, 2, 32, 0.0), (3, 1, 2, 12, 0.0), (2, 6, 3, 7, 0.05),
                                           (1, 4, 5, 5, 0.0), (1, 33, 2, 12, 0.05), (1, 64, 2, 32, 0.05),
                                           (2, 65, 2, 12, 0.0)])
def test_stitch_matches_oracle(tdm, C, T, B, o, noise):
    # tiles go through the kernel 32 at a time: T = 32, 33, 40, 64 and 65 put
    # a chunk boundary at the end, before a single tile, inside, between two
    # full chunks, and before a last single tile
    X, _, _ = synth.tile_coords(T * 7 + B, C, T, B, overlap=o, noise=noise)
    got, res = _run(tdm, X, T, o)
    ref, rref = ostitch.stitch(X.astype(np.float64), o)
    # float32 composition drifts with the number of seams: the first 40 tiles
    # at TOL_CHAIN, a longer chain as a whole at 5 TOL_CHAIN (a wrong map or
    # bead at a chunk boundary would be off by the tiles' extent)
    L40 = 64 + 39 * (64 - o)
    scale = np.abs(ref[..., :L40, :]).max(axis=(-1, -2))
    err = (np.abs(got[..., :L40, :] - ref[..., :L40, :]).max(axis=(-1, -2)) / scale).max()
    assert err <= TOL_CHAIN, err
    whole = (np.abs(got - ref).max(axis=(-1, -2)) / np.abs(ref).max(axis=(-1, -2))).max()
    assert whole <= (TOL_CHAIN if T <= 40 else 5 * TOL_CHAIN), whole
    if T > 1 and noise == 0:
        # noise-free tiles: both residuals are float32 rounding of the
        # coordinates (true value 0)
        assert res.max() <= 2e-5 * float(np.abs(X).max()) and rref.max() <= 2e-5 * float(np.abs(X).max())
    elif T > 1:
        rel = np.abs(res - rref) / np.maximum(rref, 1e-3 * noise)
        assert rel.max() <= TOL_RESID, rel.max()


def test_stitch_chromosome_chain_full_size(tdm):
    # 32 tiles x 1000 samples: every sample's chain on the GPU, 6 sampled
    # chains through the oracle
    C, T, B = 1, 32, 1000
    X, _, _ = synth.tile_coords(99, C, T, B, noise=0.02)
    got, res = _run(tdm, X, T, 12)
    assert np.isfinite(got).all() and np.isfinite(res).all()
    idx = np.random.default_rng(0).choice(B, size=6, replace=False)
    ref, rref = ostitch.stitch(X[:, :, idx].astype(np.float64))
    scale = np.abs(ref).max(axis=(-1, -2))
    assert (np.abs(got[:, idx] - ref).max(axis=(-1, -2)) / scale).max() <= TOL_CHAIN
    assert (np.abs(res[:, idx] - rref) / np.maximum(rref, 2e-5)).max() <= TOL_RESID


def test_stitch_many_pairs(tdm):
    # 4000 samples of a 32-tile chain: several waves of the kernel's CTAs;
    # chains at the start, the middle and the end through the oracle
    C, T, B = 1, 32, 4000
    X, _, _ = synth.tile_coords(7, C, T, B, noise=0.02)
    got, res = _run(tdm, X, T, 12)
    idx = np.array([0, 1, 3155, 3156, 3157, 3158, 3999])
    ref, rref = ostitch.stitch(X[:, :, idx].astype(np.float64))
    scale = np.abs(ref).max(axis=(-1, -2))
    assert (np.abs(got[:, idx] - ref).max(axis=(-1, -2)) / scale).max() <= TOL_CHAIN
    assert (np.abs(res[:, idx] - rref) / np.maximum(rref, 2e-5)).max() <= TOL_RESID


def test_stitch_long_chains_over_many_tile_chunks(tdm):
    # 520-tile chains for 400 samples: each CTA walks 17 chunks of 32 tiles,
    # carrying the composed map and the last tile's beads from chunk to chunk
    # (520 = 16 x 32 + 8, so the last chunk is ragged).  Sampled chains go
    # through the oracle: every seam's residual, and the first 40 tiles of the
    # chain (float32 composition over hundreds of seams drifts by about 1e-4
    # of the chain's extent, as test_stitch_longest_chains notes)
    C, T, B, o = 1, 520, 400, 12
    X, _, _ = synth.tile_coords(17, C, T, B, overlap=o, noise=0.02)
    got, res = _run(tdm, X, T, o)
    assert np.isfinite(got).all() and np.isfinite(res).all()
    idx = np.array([0, 193, 194, 387, 388, 399])
    ref, rref = ostitch.stitch(X[:, :, idx].astype(np.float64), o)
    L40 = 64 + 39 * (64 - o)
    scale = np.abs(ref[:, :, :L40]).max(axis=(-1, -2))
    assert (np.abs(got[:, idx, :L40] - ref[:, :, :L40]).max(axis=(-1, -2)) / scale).max() <= TOL_CHAIN
    assert (np.abs(res[:, idx] - rref) / np.maximum(rref, 2e-5)).max() <= TOL_RESID
    whole = (np.abs(got[:, idx] - ref).max(axis=(-1, -2)) / np.abs(ref).max(axis=(-1, -2))).max()
    assert whole <= 5 * TOL_CHAIN, whole


def test_stitch_longest_chains(tdm):
    # two samples of a chain of 65,535 tiles (the most a chain may have), 2048
    # chunks of tiles each.  float32 composition over 65,534 seams drifts, so the
    # oracle checks the first 40 tiles and sampled seams, and every bond of
    # both chains is checked against the walk
    C, T, B, o = 1, 65535, 2, 12
    X, walks, _ = synth.tile_coords(3, C, T, B, noise=0.0)
    got, res = _run(tdm, X, T, o)
    assert np.isfinite(got).all()
    L40 = 64 + 39 * 52
    ref, _ = ostitch.stitch(X[:, :40].astype(np.float64), o)
    for b in range(B):
        assert np.abs(got[0, b, :L40] - ref[0, b]).max() / np.abs(ref[0, b]).max() <= TOL_CHAIN
        for k in np.random.default_rng(b).choice(T - 1, 30, replace=False):
            _, _, r = ostitch.procrustes(X[0, k, b, 52:].astype(np.float64), X[0, k + 1, b, :o].astype(np.float64))
            assert abs(res[0, b, k] - r) <= 2e-5 * float(np.abs(X[0, k, b]).max())
        bond = np.linalg.norm(np.diff(got[0, b], axis=0), axis=1)
        walk_bond = np.linalg.norm(np.diff(walks[0, b], axis=0), axis=1)
        assert np.abs(bond - walk_bond).max() <= 0.05
