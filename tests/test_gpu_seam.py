"""GPU parity of the overlap projection and the seam discrepancy."""
import numpy as np
import pytest

import synth
from oracle import seam as oseam
from tests.gpu_util import TOL_SEAM, dev, host, needs_gpu, torch

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


def _rand(C, T, B, seed=0, sym=True):
    x = np.random.default_rng(seed).standard_normal((C, T, B, 64, 64)) * 5.0 + 10.0
    if sym:
        x = x + np.swapaxes(x, -1, -2)
    return x.astype(np.float32)


@pytest.mark.parametrize("o", [1, 5, 12, 32])
def test_projection_matches_oracle_exactly(tdm, o):
    x = _rand(2, 4, 3, o)
    t = tdm.Tiling(C=2, T=4, B=3, overlap=o)
    d = dev(x).reshape(-1)
    tdm.seam_project(d, t)
    g = host(d).reshape(x.shape)
    ref = oseam.seam_project(x.astype(np.float64), o)
    # 0.5f * (a + b) in float32 vs (a + b) / 2 in float64: one rounding
    np.testing.assert_allclose(g, ref, rtol=1e-7, atol=0)
    # idempotent, bit for bit
    before = d.clone()
    tdm.seam_project(d, t)
    torch.testing.assert_close(d, before, rtol=0, atol=0)
    np.testing.assert_array_equal(g[:, :-1, :, 64 - o:, 64 - o:], g[:, 1:, :, :o, :o])


def _disc_check(tdm, x, o, B):
    C, T = x.shape[:2]
    t = tdm.Tiling(C=C, T=T, B=B, overlap=o)
    out = torch.empty(C * (T - 1), device="cuda")
    tdm.seam_discrepancy(dev(x).reshape(-1), t, out)
    ref = oseam.seam_discrepancy(x.astype(np.float64), o)
    g = host(out).reshape(C, T - 1)
    floor = 1e-6 * np.abs(x).mean()
    err = np.abs(g - ref) / np.maximum(np.abs(ref), floor)
    assert err.max() <= TOL_SEAM, err.max()
    return g, ref


@pytest.mark.parametrize("C,T,B,o", [(3, 5, 1, 12), (2, 4, 7, 5), (1, 32, 200, 12), (1, 3, 1000, 32)])
def test_discrepancy_matches_oracle(tdm, C, T, B, o):
    # B = 200 and 1000 on few seams take the chunked path (partial sums in scratch)
    x = np.random.default_rng(B).standard_normal((C, T, B, 64, 64)).astype(np.float32)
    _disc_check(tdm, x, o, B)


def test_discrepancy_is_zero_after_projection(tdm):
    x = _rand(2, 6, 40, 3)
    t = tdm.Tiling(C=2, T=6, B=40, overlap=12)
    d = dev(x).reshape(-1)
    tdm.seam_project(d, t)
    out = torch.empty(10, device="cuda")
    tdm.seam_discrepancy(d, t, out)
    assert torch.all(out == 0)


def test_sharded_sums_add_up(tdm):
    x = np.random.default_rng(7).standard_normal((2, 4, 12, 64, 64)).astype(np.float32)
    ref = oseam.seam_discrepancy(x.astype(np.float64))
    total = torch.zeros(2 * 3 * 144, device="cuda")
    for b0, nb in ((0, 5), (5, 7)):
        part = dev(x[:, :, b0:b0 + nb]).reshape(-1)
        t = tdm.Tiling(C=2, T=4, B=nb, B_total=12, b_offset=b0)
        sums = torch.empty_like(total)
        tdm.seam_overlap_sums(part, t, sums)
        total += sums
    out = torch.empty(6, device="cuda")
    tdm.seam_discrepancy_finalize(total, tdm.Tiling(C=2, T=4, B=12), out)
    np.testing.assert_allclose(host(out).reshape(2, 3), ref, rtol=TOL_SEAM)
