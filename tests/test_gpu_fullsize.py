"""GPU parity at the workloads' full sizes, on sampled outputs.

The full-size GPU runs use the same launches the library makes for any size.
The oracle checks them (a) by whole oracle trajectories of sampled chains or
trajectories, and (b) for every sampled map by the closed form of the final
state that the oracle's own run is pinned to (tests/test_oracle_ddim.py): with
the ideal denoiser the last step returns x0 - c0 * (noise part of eps at step
0), c0 = sqrt(1 - ab_0) / sqrt(ab_0), then the projection.
"""
import multiprocessing as mp

import numpy as np
import pytest

import synth
from oracle import mds as omds, philox, schedule as osched, seam as oseam
from oracle.ddim import ddim_run as o_run, sample_ids, stream_noise
from tests.gpu_util import TOL_MAP, TOL_RECOVER, TOL_SEAM, assert_maps_close, dev, host, needs_gpu, normwise, torch

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


def closed_form_final(x0, g, seed, w, s_c, s_u, project, overlap=12):
    """x0 [C][T][64][64]; g [C][T][Bs] noise ids -> final maps [C][T][Bs][64][64]."""
    c0 = np.sqrt(1e-4 / (1 - 1e-4))
    noise = (1 + w) * s_c * stream_noise(seed, philox.TAG_EPS_C, 0, g)
    if w != 0:
        noise -= w * s_u * stream_noise(seed, philox.TAG_EPS_U, 0, g)
    out = x0[:, :, None].astype(np.float64) - c0 * noise
    return oseam.seam_project(out, overlap) if project else out


@pytest.mark.parametrize("eta", [0.0, 1.0])
def test_step_sweep_chain32_b100(tdm, eta):
    # 32-tile chain x 100 samples at 50, 100, 250, 500 and 1000 DDIM steps
    wl = synth.WORKLOADS["chain32_b100_sweep"]
    x0 = synth.chain_x0(wl.seed, 1, 32)
    t = tdm.Tiling(C=1, T=32, B=100, overlap=12, sync_every=1)
    maps = torch.empty(t.n_maps * 4096, device="cuda")
    rng = np.random.default_rng(int(eta))
    b_check = np.sort(rng.choice(100, size=6, replace=False))
    for S in wl.extra["S"]:
        sch = tdm.Schedule(S, eta=eta)
        tdm.ddim_run(sch, maps, dev(x0), wl.w, wl.s_c, wl.s_u, wl.seed, t)
        g = host(maps).reshape(1, 32, 100, 64, 64)
        assert np.isfinite(g).all()
        ref = closed_form_final(x0, sample_ids(1, 32, b_check, 100), wl.seed, wl.w, wl.s_c, wl.s_u, True)
        assert_maps_close(g[:, :, b_check], ref, TOL_MAP, f"S={S} closed form")
        if S == 50:
            full, traj = o_run(x0, osched.Schedule(S=S, eta=eta), wl.w, wl.s_c, wl.s_u, wl.seed,
                               [int(b_check[0])], 100, return_trajectory=True)
            assert_maps_close(g[:, :, b_check[:1]], full, TOL_MAP, f"S={S} oracle run")
            # the state before the last step, which alone sets the final maps
            tdm.ddim_run(sch, maps, dev(x0), wl.w, wl.s_c, wl.s_u, wl.seed, t, first_step=S - 1, n_steps=S - 1)
            g = host(maps).reshape(1, 32, 100, 64, 64)
            assert_maps_close(g[:, :, b_check[:1]], traj[S - 2], TOL_MAP, f"S={S} oracle run, {S - 1} steps")


def test_genome_untiled_chunked(tdm):
    # 2658 regions x {w=0, w=1} x 256 samples = 1,360,896 trajectories,
    # 50 steps, no seams, processed in chunks of 2^16 maps
    wl = synth.WORKLOADS["genome2658_b256_untiled"]
    R, B, S = wl.C, wl.B, wl.S
    chunk_regions = wl.extra["chunk_maps"] // B                      # 256 regions = 65,536 maps
    sch = tdm.Schedule(S)
    maps = torch.empty(chunk_regions * B * 4096, device="cuda")
    rng = np.random.default_rng(7)
    checked = 0
    for gi, w in enumerate(wl.extra["w"]):
        for r0 in range(0, R, chunk_regions):
            nr = min(chunk_regions, R - r0)
            x0 = synth.region_x0(wl.seed, np.arange(r0, r0 + nr))           # [nr][1][64][64]
            # the two guidance settings are separate runs of the same task
            # grid; their noise ids do not overlap
            base = gi * R * B + r0 * B
            t = tdm.Tiling(C=nr, T=1, B=B, overlap=0, sync_every=0, sample_id_base=base)
            tdm.ddim_run(sch, maps, dev(x0), w, wl.s_c, wl.s_u, wl.seed, t)
            g = maps[: nr * B * 4096].view(nr, B, 64, 64)
            assert torch.isfinite(g).all()
            # closed form on 8 random trajectories of every chunk
            cr = rng.integers(0, nr, size=8)
            cb = rng.integers(0, B, size=8)
            ids = (base + cr * B + cb).astype(np.uint64).reshape(8, 1, 1)
            ref = closed_form_final(x0[cr], ids, wl.seed, w, wl.s_c, wl.s_u, False)
            got = host(g[torch.from_numpy(cr).cuda(), torch.from_numpy(cb).cuda()]).reshape(8, 1, 1, 64, 64)
            assert_maps_close(got, ref, TOL_MAP, f"w={w} regions {r0}..")
            checked += 8
            if r0 == 0:
                # a whole oracle trajectory of one sample of the chunk's first region
                full = o_run(x0[:1], osched.Schedule(S=S), w, wl.s_c, wl.s_u, wl.seed, [3], B,
                             sync_every=0, sample_id_base=base)
                assert_maps_close(host(g[0, 3]).reshape(1, 1, 1, 64, 64), full, TOL_MAP, "oracle run")
    assert checked == 2 * 11 * 8


def test_recovery_1m(tdm):
    # 1,000,000 noisy point-cloud maps: MDS, reconstruction, Eq. (6) over
    # 31,250 chains x 32 tiles x 1 sample
    n = 1_000_000
    maps = torch.empty(n * 4096, device="cuda")
    view = maps.view(n, 4096)
    nblk = -(-n // synth.CLOUD_BLOCK)
    with mp.get_context("spawn").Pool(min(16, max(2, mp.cpu_count()))) as pool:
        for blk, arr in pool.imap_unordered(synth.cloud_block_maps, range(nblk), chunksize=4):
            lo = blk * synth.CLOUD_BLOCK
            hi = min(n, lo + synth.CLOUD_BLOCK)
            view[lo:hi].copy_(torch.from_numpy(arr[: hi - lo].reshape(hi - lo, 4096)))
    coords = torch.empty(n * 192, device="cuda")
    eig = torch.empty(n * 3, device="cuda")
    rec = torch.empty(n * 4096, device="cuda")
    disc = torch.empty(31250 * 31, device="cuda")
    t = tdm.Tiling(C=31250, T=32, B=1, overlap=12, sync_every=0)
    tdm.mds_recover(maps, n, coords, eig)
    tdm.pairwise_dist(coords, n, rec)
    tdm.seam_discrepancy(rec, t, disc)
    flags = tdm.ctx_sync()
    assert flags == 0, "MDS reported non-convergence"
    assert torch.isfinite(rec).all() and torch.isfinite(disc).all()
    # sampled maps: the oracle's recovery of the same inputs
    rng = np.random.default_rng(11)
    idx = np.sort(rng.choice(n, size=48, replace=False))
    inp = np.stack([synth.cloud_maps(0, int(i), 1)[0] for i in idx])
    Xo, lo = omds.classical_mds(inp.astype(np.float64))
    Ro = omds.pairwise_distances(Xo)
    got = host(rec.view(n, 64, 64)[torch.from_numpy(idx).cuda()])
    e = normwise(got, Ro)
    assert e.max() <= TOL_RECOVER, e.max()
    lam = host(eig.view(n, 3)[torch.from_numpy(idx).cuda()])
    assert (np.abs(lam - lo[:, :3]).max(axis=1) / lo[:, 0]).max() <= TOL_RECOVER
    # sampled seams: one whole chain through the oracle pipeline
    c = int(rng.integers(0, 31250))
    chain = synth.cloud_maps(0, c * 32, 32).astype(np.float64)
    Xc, _ = omds.classical_mds(chain)
    Rc = omds.pairwise_distances(Xc).reshape(1, 32, 1, 64, 64)
    d_ref = oseam.seam_discrepancy(Rc)[0]
    d_got = host(disc.view(31250, 31)[c])
    # Eq. (6) of reconstructed maps differs by at most the reconstruction
    # error of the two blocks it compares
    rec_err = np.abs(host(rec.view(n, 64, 64)[c * 32:(c + 1) * 32]) - Rc.reshape(32, 64, 64)).max()
    assert np.all(np.abs(d_got - d_ref) <= 2 * rec_err + TOL_SEAM * np.abs(d_ref))
