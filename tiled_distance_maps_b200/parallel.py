"""Sample sharding across GPUs (one process per GPU, torch.distributed).

The sampler's tasks never communicate while denoising (ParaChromo,
mdpi.com/2079-9292/15/13/2750, §3.3 and §4.1), and the projection couples
only tiles of the same sample (§4.3.2).  So a joint run of B_total samples is
split by sample index: every rank holds all tiles of its samples, and the
noise ids (global sample indices) make each rank's maps equal to the same
slice of the unsplit run.  The only exchange is the seam discrepancy of
Eq. (6), whose per-sample mean spans all ranks: one all-reduce of the
per-seam overlap sums, between tdm_seam_overlap_sums and
tdm_seam_discrepancy_finalize.
"""
from __future__ import annotations

from dataclasses import replace


def shard_range(B_total: int, rank: int, world: int) -> tuple[int, int]:
    """(b_offset, B) of this rank: contiguous, sizes differing by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    base, extra = divmod(B_total, world)
    b_offset = rank * base + min(rank, extra)
    return b_offset, base + (1 if rank < extra else 0)


def shard_tiling(tiling, rank: int, world: int):
    """The tiling of this rank's samples (a ``Tiling`` whose B is the global
    sample count, or whose B_total is set)."""
    B_total = tiling.B_total or tiling.B
    b_offset, B = shard_range(B_total, rank, world)
    return replace(tiling, B=B, B_total=B_total, b_offset=tiling.b_offset + b_offset)


def allreduce_sums(sums, group=None):
    """Sum the per-seam overlap sums over all ranks (in place)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(sums, op=dist.ReduceOp.SUM, group=group)
    return sums


def sharded_seam_discrepancy(maps, tiling, sums, out, group=None, ctx=None):
    """Eq. (6) of a run whose samples are split over the ranks of ``group``:
    local overlap sums (GPU), all-reduce, then the finalisation (GPU) with
    the global sample count."""
    from . import seam_discrepancy_finalize, seam_overlap_sums
    seam_overlap_sums(maps, tiling, sums, ctx=ctx)
    allreduce_sums(sums, group)
    seam_discrepancy_finalize(sums, tiling, out, ctx=ctx)
    return out
