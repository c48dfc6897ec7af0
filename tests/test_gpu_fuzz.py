"""Seeded random configurations of the fused run against the float64 oracle:
chains, tiles, samples, overlap (multiple of 4), projection interval, step
count, eta, guidance weight and the noise scales, with sample shards (b_offset,
B_total) and noise-id offsets, at sizes the oracle finishes in a second.  Half
the configurations perturb x0 so that tile overlaps disagree; each compares the
final maps and one state before the last step."""
import numpy as np
import pytest

import synth
from oracle import schedule as osched
from oracle.ddim import ddim_run as o_run
from tests.gpu_util import TOL_MAP, assert_maps_close, dev, host, needs_gpu, torch

pytestmark = [pytest.mark.gpu, needs_gpu]

STEPS = [1, 2, 4, 5, 8, 10, 20, 25, 40, 50]


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


def _config(k):
    g = np.random.default_rng([2024, k])
    T = int(g.integers(1, 6))
    cfg = dict(C=int(g.integers(1, 4)), T=T, B=int(g.integers(1, 6)), overlap=int(4 * g.integers(1, 9)),
               K=int(g.choice([0, 1, 2, 3, 7])), S=int(g.choice(STEPS)), eta=float(g.choice([0.0, 0.5, 1.0])),
               w=float(g.choice([0.0, 0.5, 1.0, 3.0])), s_c=float(g.uniform(0.0, 0.5)),
               s_u=float(g.uniform(0.0, 0.5)), seed=int(g.integers(0, 2 ** 63)), base=int(g.integers(0, 1000)),
               init=bool(g.integers(0, 2)))
    cfg["extra"] = int(g.integers(0, 3))      # samples of the joint run held by other shards
    cfg["boff"] = int(g.integers(0, cfg["extra"] + 1))
    return cfg


@pytest.mark.parametrize("k", range(64))
def test_random_fused_runs(tdm, k):
    c = _config(k)
    C, T, B, o = c["C"], c["T"], c["B"], c["overlap"]
    B_total = B + c["extra"]
    t = tdm.Tiling(C=C, T=T, B=B, overlap=o, sync_every=c["K"], B_total=B_total, b_offset=c["boff"],
                   sample_id_base=c["base"])
    x0 = synth.chain_x0(k, C, T, overlap=o) * float(1 + k % 3)
    if k % 2:   # overlaps that disagree between tiles
        p = np.random.default_rng([k, 505]).uniform(-0.5, 0.5, size=x0.shape)
        x0 = (x0 + 0.5 * (p + np.swapaxes(p, -1, -2))).astype(np.float32)
    sch = tdm.Schedule(c["S"], eta=c["eta"])
    b_index = np.arange(c["boff"], c["boff"] + B)
    if c["init"]:
        maps = torch.empty(t.n_maps * 4096, device="cuda")
        x_T = None
    else:
        x_T = synth.gaussian_maps(k + 100, C * T * B).reshape(C, T, B, 64, 64) * 2.0
        maps = dev(x_T).reshape(-1).clone()
    start = maps.clone()
    tdm.ddim_run(sch, maps, dev(x0), c["w"], c["s_c"], c["s_u"], c["seed"], t, init_noise=c["init"])
    ref, traj = o_run(x0, osched.Schedule(S=c["S"], eta=c["eta"]), c["w"], c["s_c"], c["s_u"], c["seed"], b_index,
                      B_total, overlap=o, sync_every=c["K"], sample_id_base=c["base"], x_T=x_T,
                      return_trajectory=True)
    got = host(maps).reshape(C, T, B, 64, 64)
    assert_maps_close(got, ref, TOL_MAP, f"config {c}")
    if c["S"] > 1:
        # a state before the last step (the last step alone sets the final maps)
        m = 1 + k % (c["S"] - 1)
        tdm.ddim_run(sch, start, dev(x0), c["w"], c["s_c"], c["s_u"], c["seed"], t, init_noise=c["init"],
                     first_step=c["S"] - 1, n_steps=m)
        assert_maps_close(host(start).reshape(C, T, B, 64, 64), traj[m - 1], TOL_MAP, f"config {c}, {m} steps")


@pytest.mark.parametrize("k", range(24))
def test_random_per_step_runs(tdm, k):
    # the per-step path (stand-in eps, DDIM step, projection when due), which
    # also takes overlaps that are not a multiple of 4
    from tests.test_gpu_sampler import _gpu_per_step
    g = np.random.default_rng([4048, k])
    C, T, B = int(g.integers(1, 3)), int(g.integers(1, 5)), int(g.integers(1, 4))
    o = int(g.integers(1, 33))
    K, S = int(g.choice([0, 1, 2, 3])), int(g.choice([1, 2, 4, 5, 8, 10]))
    eta, w = float(g.choice([0.0, 1.0])), float(g.choice([0.0, 1.0, 2.0]))
    seed = int(g.integers(0, 2 ** 40))
    t = tdm.Tiling(C=C, T=T, B=B, overlap=o, sync_every=K)
    x0 = synth.chain_x0(k, C, T, overlap=o)
    got = _gpu_per_step(tdm, tdm.Schedule(S, eta=eta), x0, t, w, 0.1, 0.3, seed)[-1]
    ref = o_run(x0, osched.Schedule(S=S, eta=eta), w, 0.1, 0.3, seed, np.arange(B), B, overlap=o, sync_every=K)
    assert_maps_close(got, ref, TOL_MAP, f"per-step C={C} T={T} B={B} o={o} K={K} S={S} eta={eta} w={w}")
