"""The pipeline of entry points captured in a CUDA graph: after warm-up calls
(which build the lane plan and the cached launch shapes) every entry point of
the step is capturable, and replays reproduce the direct calls bit for bit."""
import numpy as np
import pytest

import synth
from tests.gpu_util import dev, host, needs_gpu, torch

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


def test_step_replays_from_a_cuda_graph(tdm):
    C, T, B = 1, 4, 8
    t = tdm.Tiling(C=C, T=T, B=B, overlap=12, sync_every=1)
    n = t.n_maps
    sch = tdm.Schedule(50)
    x0 = dev(synth.chain_x0(0, C, T)).reshape(-1)
    maps, coords = torch.empty(n * 4096, device="cuda"), torch.empty(n * 192, device="cuda")
    rec, disc = torch.empty(n * 4096, device="cuda"), torch.empty(C * (T - 1), device="cuda")
    chains = torch.empty(C * B * (64 + (T - 1) * 52) * 3, device="cuda")

    def step(seed):
        tdm.ddim_run(sch, maps, x0, 1.0, 0.1, 0.3, seed, t)
        tdm.mds_recover(maps, n, coords)
        tdm.refine_smacof(maps, n, coords, 5)
        tdm.pairwise_dist(coords, n, rec)
        tdm.seam_discrepancy(rec, t, disc)
        tdm.kabsch_stitch(coords, t, chains)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step(7)                                  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    direct = [host(v).copy() for v in (maps, coords, rec, disc, chains)]
    for v in (maps, coords, rec, disc, chains):
        v.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(7)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for d, v in zip(direct, (maps, coords, rec, disc, chains)):
        np.testing.assert_array_equal(host(v), d)
    assert tdm.ctx_sync() == 0
