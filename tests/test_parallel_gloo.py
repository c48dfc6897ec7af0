"""The multi-GPU host logic on CPU: world size 2 over gloo.

Each rank takes its shard of the samples through the product's
``parallel.shard_tiling``, runs the sampler on it, and computes Eq. (6) through
the product's ``parallel.sharded_seam_discrepancy`` (overlap sums, the
``allreduce_sums`` all-reduce, finalisation).  The two GPU halves of that
wrapper are replaced by the float64 oracle on CPU tensors, since the kernels
need a GPU; the sharding and the collective are the product's own code.  The
result must equal the unsplit run: the maps of each shard bit for bit, Eq. (6)
to rounding.
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
    import tiled_distance_maps_b200 as tdm
    from oracle import schedule, seam
    from oracle.ddim import ddim_run
    from tiled_distance_maps_b200 import parallel
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        C, T, B_total = 2, 3, 6
        t = parallel.shard_tiling(tdm.Tiling(C=C, T=T, B=B_total, overlap=12), rank, world)
        assert t.B_total == B_total
        x0 = synth.chain_x0(3, C, T)
        out = ddim_run(x0, schedule.Schedule(S=4), 1.0, 0.1, 0.3, 11,
                       np.arange(t.b_offset, t.b_offset + t.B), B_total)

        # the kernels' halves of the wrapper, on CPU tensors through the oracle
        def overlap_sums(maps, tiling, sums, ctx=None):
            sums.copy_(torch.from_numpy(seam.overlap_difference_sums(maps)).reshape(sums.shape))

        def finalize(sums, tiling, o, ctx=None):
            shape = (tiling.C, tiling.T - 1, tiling.overlap, tiling.overlap)
            o.copy_(torch.from_numpy(seam.discrepancy_from_sums(sums.numpy().reshape(shape),
                                                                 tiling.B_total)).reshape(o.shape))

        tdm.seam_overlap_sums, tdm.seam_discrepancy_finalize = overlap_sums, finalize
        sums = torch.empty(C * (T - 1) * 12 * 12, dtype=torch.float64)
        disc = torch.empty(C * (T - 1), dtype=torch.float64)
        parallel.sharded_seam_discrepancy(out, t, sums, disc)
        q.put((rank, t.b_offset, out, disc.numpy().reshape(C, T - 1)))
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
