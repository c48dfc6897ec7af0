"""The allocation-free seam discrepancy, checked against the regular one.

tdm_seam_discrepancy_noalloc serves callers that cannot call cudaMalloc: an
application that has handed all device memory to its own pool, a plugin host
that forbids allocations outside its allocator, or a pipeline that must not
pay the synchronisation an allocation may cause.  It keeps its partial sums in
a fixed array inside the library instead of a context's scratch.  This file
is collected last on purpose (the name), so that a run that stops at the first
failure has already run every other test; it also passes on its own.
"""
import numpy as np
import pytest

from tests.gpu_util import TOL_SEAM, dev, host, needs_gpu, torch

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


def _close(a, b, x):
    floor = 1e-6 * np.abs(x).mean()
    err = np.abs(a - b) / np.maximum(np.abs(b), floor)
    return err.max()


@pytest.mark.parametrize("C,T,B,o", [(1, 6, 400, 12), (2, 4, 200, 8), (1, 3, 400, 32), (40, 9, 2, 12),
                                     (1, 11, 500, 32)])
def test_noalloc_matches_the_regular_entry_point_twice_in_a_row(tdm, C, T, B, o):
    # the first three shapes split each seam's samples into chunks (partial
    # sums in the library's fixed array); the fourth takes the direct path; the
    # last would need 10 seams x 60 chunks x 32^2 partial sums, more than the
    # fixed array holds, so it takes the direct path too
    t = tdm.Tiling(C=C, T=T, B=B, overlap=o)
    outs = []
    for call in range(2):
        x = np.random.default_rng(100 * call + B).standard_normal((C, T, B, 64, 64)).astype(np.float32)
        d = dev(x).reshape(-1)
        ref = torch.empty(C * (T - 1), device="cuda")
        got = torch.full((C * (T - 1),), float("nan"), device="cuda")
        tdm.seam_discrepancy(d, t, ref)
        tdm.seam_discrepancy_noalloc(d, t, got)
        torch.cuda.synchronize()
        assert _close(host(got), host(ref), x) <= TOL_SEAM, f"call {call}"
        outs.append(host(got))
    # two different inputs, two different answers: nothing stale is reused
    assert not np.array_equal(outs[0], outs[1])


def test_noalloc_rejects_bad_arguments(tdm):
    m = torch.zeros(2 * 4096, device="cuda")
    out = torch.zeros(4, device="cuda")
    with pytest.raises(tdm.TdmError) as e:
        tdm.seam_discrepancy_noalloc(m, tdm.Tiling(C=1, T=1, B=2), out)
    assert e.value.status == tdm.EINVAL
    with pytest.raises(tdm.TdmError) as e:
        tdm.seam_discrepancy_noalloc(m[1:], tdm.Tiling(C=1, T=2, B=0, overlap=12), out)
    assert e.value.status == tdm.EINVAL


def test_noalloc_second_call_takes_no_device_memory(tdm):
    # the first call on a device may load the library's device code (and the
    # fixed array with it); from then on a call must leave free memory as it is
    C, T, B, o = 1, 6, 400, 12
    t = tdm.Tiling(C=C, T=T, B=B, overlap=o)
    x = np.random.default_rng(7).standard_normal((C, T, B, 64, 64)).astype(np.float32)
    d = dev(x).reshape(-1)
    out = torch.empty(C * (T - 1), device="cuda")
    tdm.seam_discrepancy_noalloc(d, t, out)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    first = host(out)
    tdm.seam_discrepancy_noalloc(d, t, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    assert np.array_equal(host(out), first)


def test_noalloc_rejects_out_on_another_device(tdm):
    m = torch.zeros(2 * 4096, device="cuda")
    with pytest.raises((ValueError, TypeError)):
        tdm.seam_discrepancy_noalloc(m, tdm.Tiling(C=1, T=2, B=1, overlap=12), torch.zeros(1))
