"""Seeded synthetic inputs shaped like the ParaChromo workloads.

This module is shared by the oracle side (tests, CPU baseline) and the CUDA side
(tests, bench).  It draws only the *inputs* of the sampler -- the reference maps
x0 that the stand-in denoiser pulls toward, and the noisy point-cloud distance
maps fed to coordinate recovery.  It holds none of the sampler's arithmetic: no
schedule, no DDIM update, no projection, no eigen-solve and none of the Philox
noise that the sampler itself draws.

Randomness comes from numpy's own generators keyed by ``(seed, tag, item)``
through ``numpy.random.SeedSequence``, so that any single chain, region or block
of maps can be regenerated on its own (the oracle checks sampled outputs one by
one at full size).

Shapes follow the ParaChromo paper (mdpi.com/2079-9292/15/13/2750):
  * a region is 64 beads at 20 kb (§3.2), adjacent regions share 12 beads
    (240 kb, §3.2), so the tile stride is 52 beads;
  * a chromosome-scale chain is 32 tiles / 31 seams / 1676 unique beads (§1, §5.5);
  * samples of one condition differ only through their noise (§3.3), so x0 is
    one map per (chain, tile), shared over the samples.
"""
from __future__ import annotations

import numpy as np

N_BEADS = 64
OVERLAP = 12

# tags separating the generator streams
_TAG_CHAIN = 0xC4A1
_TAG_REGION = 0x4E61
_TAG_CLOUD = 0xC10D

# point-cloud maps are generated in blocks of this many maps, each block from
# its own generator, so any map index can be regenerated without the others
CLOUD_BLOCK = 1024


def _rng(*words: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(w) for w in words]))


def _distance_map(p: np.ndarray) -> np.ndarray:
    """Euclidean distance matrix of bead positions ``p[..., n, 3]`` in float64."""
    d = p[..., :, None, :] - p[..., None, :, :]
    return np.sqrt(np.sum(d * d, axis=-1))


def chain_beads(n_tiles: int, overlap: int = OVERLAP, n: int = N_BEADS) -> int:
    """Unique beads covered by a chain of ``n_tiles`` tiles of ``n`` beads."""
    return n_tiles * n - (n_tiles - 1) * overlap


def chain_walk(seed: int, chain: int, n_tiles: int, overlap: int = OVERLAP,
               sigma: str = "unit") -> np.ndarray:
    """One continuous 3D Gaussian random walk covering a whole chain of tiles.

    Bond j (bead j -> j+1) has step sigma of tile ``min(j // stride, n_tiles-1)``.
    ``sigma="unit"``: every step has sigma 1.  ``sigma="tile_uniform"``: one
    sigma per tile drawn from U(0.8, 1.2).  Returns positions ``[beads, 3]``.
    """
    stride = N_BEADS - overlap
    nb = chain_beads(n_tiles, overlap)
    g = _rng(seed, _TAG_CHAIN, chain)
    if sigma == "unit":
        sig_tile = np.ones(n_tiles)
    elif sigma == "tile_uniform":
        sig_tile = g.uniform(0.8, 1.2, size=n_tiles)
    else:
        raise ValueError(f"unknown sigma mode {sigma!r}")
    bond_tile = np.minimum(np.arange(nb - 1) // stride, n_tiles - 1)
    steps = g.standard_normal((nb - 1, 3)) * sig_tile[bond_tile][:, None]
    return np.concatenate([np.zeros((1, 3)), np.cumsum(steps, axis=0)], axis=0)


def chain_x0(seed: int, n_chains: int, n_tiles: int, overlap: int = OVERLAP,
             sigma: str = "unit", chains=None) -> np.ndarray:
    """Reference maps ``x0[C][T][64][64]`` (float32) of tiled random-walk chains.

    Tile k of a chain is the distance map of beads ``[k*stride, k*stride+64)`` of
    that chain's walk, so the overlap blocks of adjacent tiles agree exactly (the
    physical consistency that the overlap equality of ParaChromo §4.3.1 states).
    ``chains`` optionally selects which chain indices to build.
    """
    stride = N_BEADS - overlap
    idx = range(n_chains) if chains is None else chains
    out = []
    for c in idx:
        p = chain_walk(seed, c, n_tiles, overlap, sigma)
        tiles = np.stack([p[k * stride:k * stride + N_BEADS] for k in range(n_tiles)])
        out.append(_distance_map(tiles))
    return np.asarray(out, dtype=np.float32).reshape(len(out), n_tiles, N_BEADS, N_BEADS)


def region_x0(seed: int, regions) -> np.ndarray:
    """Reference maps ``x0[R][1][64][64]`` (float32) for independent regions.

    Each region is one 64-bead walk with unit step sigma, seeded by its region
    index (the genome-wide untiled workload: 2658 regions, ParaChromo §3.1).
    """
    regions = np.atleast_1d(np.asarray(regions, dtype=np.int64))
    out = np.empty((len(regions), 1, N_BEADS, N_BEADS), dtype=np.float32)
    for i, r in enumerate(regions):
        g = _rng(seed, _TAG_REGION, int(r))
        steps = g.standard_normal((N_BEADS - 1, 3))
        p = np.concatenate([np.zeros((1, 3)), np.cumsum(steps, axis=0)], axis=0)
        out[i, 0] = _distance_map(p)
    return out


def cloud_block(seed: int, block: int, noise: float = 0.01):
    """One block of ``CLOUD_BLOCK`` noisy point-cloud distance maps.

    Points: 64 per map, N(0, sigma^2 I3) with sigma ~ U(1, 10) per map.
    Noise: multiplicative, D_ij * (1 + noise * z_ij) for i < j, mirrored, zero
    diagonal.  Returns ``(maps float32 [CLOUD_BLOCK,64,64], points float64
    [CLOUD_BLOCK,64,3], sigma float64 [CLOUD_BLOCK])``.
    """
    g = _rng(seed, _TAG_CLOUD, block)
    sig = g.uniform(1.0, 10.0, size=CLOUD_BLOCK)
    pts = g.standard_normal((CLOUD_BLOCK, N_BEADS, 3)) * sig[:, None, None]
    z = g.standard_normal((CLOUD_BLOCK, N_BEADS, N_BEADS))
    d = _distance_map(pts)
    iu = np.triu(np.ones((N_BEADS, N_BEADS), dtype=bool), 1)
    f = np.where(iu, 1.0 + noise * z, 0.0)
    f = f + np.swapaxes(f, -1, -2)
    return (d * f).astype(np.float32), pts, sig


def cloud_block_maps(block: int, seed: int = 0, noise: float = 0.01):
    """``(block, maps)`` of one block (for process pools)."""
    return block, cloud_block(seed, block, noise)[0]


def cloud_maps(seed: int, start: int, count: int, noise: float = 0.01) -> np.ndarray:
    """Maps ``[start, start+count)`` of the point-cloud recovery workload."""
    out = np.empty((count, N_BEADS, N_BEADS), dtype=np.float32)
    pos = 0
    while pos < count:
        m = start + pos
        blk, off = divmod(m, CLOUD_BLOCK)
        maps, _, _ = cloud_block(seed, blk, noise)
        take = min(CLOUD_BLOCK - off, count - pos)
        out[pos:pos + take] = maps[off:off + take]
        pos += take
    return out


def random_orthogonal(g: np.random.Generator, proper: bool = False) -> np.ndarray:
    """A random 3x3 orthogonal matrix (det -1 half of the time unless proper)."""
    q, r = np.linalg.qr(g.standard_normal((3, 3)))
    q = q * np.sign(np.diag(r))
    if proper and np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q


def tile_coords(seed: int, n_chains: int, n_tiles: int, n_samples: int, overlap: int = OVERLAP,
                noise: float = 0.0, proper: bool = False):
    """Per-tile coordinates ``[C][T][B][64][3]`` (float32) of random-walk chains.

    Sample b of chain c is one walk of the chain's length; tile k holds beads
    [k*stride, k*stride + 64) under its own random orthogonal map (improper
    half of the time unless ``proper``) and translation, plus ``noise`` N(0,1)
    per coordinate -- the shape of per-tile recovered coordinates.  Also
    returns the walks ``[C][B][L][3]`` (float64) and the tile maps
    ``(R [C][T][B][3][3], t [C][T][B][3])`` (tile beads = R @ walk + t).
    """
    stride = N_BEADS - overlap
    L = chain_beads(n_tiles, overlap)
    out = np.empty((n_chains, n_tiles, n_samples, N_BEADS, 3), dtype=np.float32)
    walks = np.empty((n_chains, n_samples, L, 3))
    Rs = np.empty((n_chains, n_tiles, n_samples, 3, 3))
    ts = np.empty((n_chains, n_tiles, n_samples, 3))
    for c in range(n_chains):
        for b in range(n_samples):
            g = _rng(seed, 0x57C4, c, b)
            steps = g.standard_normal((L - 1, 3))
            w = np.concatenate([np.zeros((1, 3)), np.cumsum(steps, axis=0)], axis=0)
            walks[c, b] = w
            for k in range(n_tiles):
                R = random_orthogonal(g, proper)
                t = g.standard_normal(3) * 10.0
                x = w[k * stride:k * stride + N_BEADS] @ R.T + t
                if noise:
                    x = x + noise * g.standard_normal(x.shape)
                out[c, k, b] = x
                Rs[c, k, b], ts[c, k, b] = R, t
    return out, walks, (Rs, ts)


def random_points(seed: int, count: int, n: int = N_BEADS, scale: float = 1.0) -> np.ndarray:
    """``[count, n, 3]`` float64 Gaussian points (for exact-distance checks)."""
    return _rng(seed, 0x9017, count, n).standard_normal((count, n, 3)) * scale


def exact_distance_maps(points: np.ndarray) -> np.ndarray:
    """Exact Euclidean distance maps of ``points[..., n, 3]`` in float64."""
    return _distance_map(points)


def gaussian_maps(seed: int, count: int, symmetric: bool = True) -> np.ndarray:
    """``[count, 64, 64]`` float32 N(0,1) maps (e.g. a caller-supplied x_T)."""
    z = _rng(seed, 0x6A55, count).standard_normal((count, N_BEADS, N_BEADS))
    if symmetric:
        z = np.triu(z) + np.swapaxes(np.triu(z, 1), -1, -2)
    return z.astype(np.float32)


from .workloads import WORKLOADS, Workload  # noqa: E402,F401
