"""The multi-GPU host logic on CPU: world size 2 over gloo.

Each rank takes its shard of the samples, runs the sampler and Eq. (6)'s
overlap sums on it (the float64 oracle stands in for the kernels here, since
the kernels need a GPU), all-reduces the sums and finalises.  The result must
equal the unsplit run: the maps of each shard bit for bit, Eq. (6) to
rounding.
"""
import os
import socket

import numpy as np
import pytest

from tiled_distance_maps_b200.parallel import shard_range, shard_tiling


def test_shard_ranges_cover_the_samples():
    for B, world in ((1000, 2), (1000, 3), (7, 4), (3, 5)):
        got = [shard_range(B, r, world) for r in range(world)]
        assert sum(n for _, n in got) == B
        assert [o for o, _ in got] == list(np.cumsum([0] + [n for _, n in got[:-1]]))
        assert max(n for _, n in got) - min(n for _, n in got) <= 1


def test_shard_tiling_keeps_global_ids():
    import tiled_distance_maps_b200 as tdm
    t = tdm.Tiling(C=1, T=32, B=1000)
    s = shard_tiling(t, 1, 2)
    assert (s.B, s.B_total, s.b_offset) == (500, 1000, 500)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import synth
    from oracle import schedule, seam
    from oracle.ddim import ddim_run
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        C, T, B_total = 2, 3, 6
        b0, nb = shard_range(B_total, rank, world)
        x0 = synth.chain_x0(3, C, T)
        out = ddim_run(x0, schedule.Schedule(S=4), 1.0, 0.1, 0.3, 11, np.arange(b0, b0 + nb), B_total)
        sums = torch.from_numpy(seam.overlap_difference_sums(out))
        dist.all_reduce(sums)
        disc = seam.discrepancy_from_sums(sums.numpy(), B_total)
        q.put((rank, b0, out, disc))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reproduce_the_unsplit_run():
    import multiprocessing as mp

    import synth
    from oracle import schedule, seam
    from oracle.ddim import ddim_run
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    x0 = synth.chain_x0(3, 2, 3)
    full = ddim_run(x0, schedule.Schedule(S=4), 1.0, 0.1, 0.3, 11, np.arange(6), 6)
    ref = seam.seam_discrepancy(full)
    for rank, b0, out, disc in res:
        np.testing.assert_array_equal(out, full[:, :, b0:b0 + out.shape[2]])
        np.testing.assert_allclose(disc, ref, rtol=1e-12)
