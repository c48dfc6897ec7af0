"""Guard bands: every entry point, on ragged sizes, writes only inside its
output buffers.  Each output is the middle of a larger buffer whose 64-float
bands on both sides hold a sentinel; the bands must be unchanged afterwards
(a bounds check of the kernels' index arithmetic that needs no sanitizer)."""
import numpy as np
import pytest

import synth
from tests.gpu_util import dev, needs_gpu, torch

pytestmark = [pytest.mark.gpu, needs_gpu]

G = 64                      # guard floats per side (256 bytes: keeps 16-byte alignment)
SENT = -7.125e30
USENT = 0xA5A5A5A5


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


class Guarded:
    def __init__(self, n, fill=None, dtype=torch.float32):
        self.n = n
        if dtype == torch.float32:
            self.buf = torch.full((n + 2 * G,), SENT, device="cuda", dtype=dtype)
        else:
            self.buf = torch.from_numpy(np.full(n + 2 * G, USENT, dtype=np.uint32)).cuda()
        self.t = self.buf[G:G + n]
        if fill is not None:
            self.t.copy_(fill.reshape(-1))

    def intact(self):
        torch.cuda.synchronize()
        h = self.buf.cpu().numpy()
        s = SENT if h.dtype == np.float32 else USENT
        return bool(np.all(h[:G] == np.asarray(s, dtype=h.dtype))) and \
            bool(np.all(h[G + self.n:] == np.asarray(s, dtype=h.dtype)))


@pytest.mark.parametrize("C,T,B,o", [(2, 3, 5, 12), (1, 1, 3, 12), (3, 2, 1, 8)])
def test_sampler_and_seam_outputs_stay_in_bounds(tdm, C, T, B, o):
    t = tdm.Tiling(C=C, T=T, B=B, overlap=o, sync_every=1)
    n = t.n_maps
    sch = tdm.Schedule(10, eta=1.0)
    x0 = dev(synth.chain_x0(1, C, T, overlap=o)).reshape(-1)
    maps = Guarded(n * 4096)
    tdm.init_noise(maps.t, t, 3)
    assert maps.intact(), "init_noise"
    ec, eu = Guarded(n * 4096), Guarded(n * 4096)
    tdm.eps_standin(sch, 5, maps.t, x0, 0.1, tdm.STREAM_EPS_C, 3, t, ec.t)
    tdm.eps_standin(sch, 5, maps.t, x0, 0.3, tdm.STREAM_EPS_U, 3, t, eu.t)
    assert ec.intact() and eu.intact(), "eps_standin"
    tdm.ddim_step(sch, 5, maps.t, ec.t, eu.t, 1.0, 3, t)
    assert maps.intact(), "ddim_step"
    tdm.seam_project(maps.t, t)
    assert maps.intact(), "seam_project"
    if T == 1 or o % 4 == 0:
        tdm.ddim_run(sch, maps.t, x0, 1.0, 0.1, 0.3, 3, t)
        tdm.ddim_run(sch, maps.t, x0, 1.0, 0.1, 0.3, 3, t, init_noise=False, first_step=4, n_steps=3)
        assert maps.intact(), "ddim_run"
    if T > 1:
        d = Guarded(C * (T - 1))
        tdm.seam_discrepancy(maps.t, t, d.t)
        assert d.intact(), "seam_discrepancy"
        sums = Guarded(C * (T - 1) * o * o)
        tdm.seam_overlap_sums(maps.t, t, sums.t)
        tdm.seam_discrepancy_finalize(sums.t, t, d.t)
        assert sums.intact() and d.intact(), "sharded seam discrepancy"
        dn = Guarded(C * (T - 1))
        tdm.seam_discrepancy_noalloc(maps.t, t, dn.t)
        assert dn.intact(), "seam_discrepancy_noalloc"
    ref = dev(synth.gaussian_maps(4, n)).reshape(-1)
    ts, ratio = Guarded(C * T * 2), Guarded(C)
    tdm.nonoverlap_drift(maps.t, ref, t, ts.t, ratio.t)
    assert ts.intact() and ratio.intact(), "nonoverlap_drift"


@pytest.mark.parametrize("n", [1, 5, 37])
def test_recovery_outputs_stay_in_bounds(tdm, n):
    maps = dev(synth.cloud_maps(0, 0, n)).reshape(-1)
    coords, eig = Guarded(n * 192), Guarded(n * 3)
    tdm.mds_recover(maps, n, coords.t, eig.t)
    assert coords.intact() and eig.intact(), "mds_recover"
    out = Guarded(n * 4096)
    tdm.pairwise_dist(coords.t, n, out.t)
    assert out.intact(), "pairwise_dist"
    stress = Guarded(n)
    tdm.refine_smacof(maps, n, coords.t, 3, stress.t)
    assert coords.intact() and stress.intact(), "refine_smacof"
    dist = Guarded(n * 4096)
    tdm.mds_reconstruct(maps, n, coords.t, dist.t, eig.t)
    assert coords.intact() and eig.intact() and dist.intact(), "mds_reconstruct"


@pytest.mark.parametrize("C,T,B,o", [(2, 3, 5, 12), (1, 1, 2, 12), (1, 4, 3, 7)])
def test_stitch_outputs_stay_in_bounds(tdm, C, T, B, o):
    X, _, _ = synth.tile_coords(1, C, T, B, overlap=o, noise=0.01)
    t = tdm.Tiling(C=C, T=T, B=B, overlap=o)
    L = 64 + (T - 1) * (64 - o)
    chain, res = Guarded(C * B * L * 3), Guarded(max(C * B * (T - 1), 1))
    tdm.kabsch_stitch(dev(X).reshape(-1), t, chain.t, res.t if T > 1 else None)
    assert chain.intact() and res.intact(), "kabsch_stitch"


def test_noise_primitives_stay_in_bounds(tdm):
    n = 37
    g = np.random.default_rng(0)
    ctr = torch.from_numpy(g.integers(0, 2 ** 32, size=4 * n, dtype=np.uint64).astype(np.uint32)).cuda()
    out = Guarded(4 * n, dtype=torch.uint32)
    tdm.philox4x32(ctr, 5, out.t)
    assert out.intact(), "philox4x32"
    z = Guarded(4 * n)             # 4n words = 2n pairs = 4n normals
    tdm.box_muller(out.t, z.t)
    assert z.intact(), "box_muller"


@pytest.mark.parametrize("n,off", [(1, 0), (4099, 1), (1 << 20, 3), (7, 2)])
def test_nonfinite_scan(tdm, n, off):
    # a clean buffer raises nothing; one NaN or inf anywhere (head, body or
    # tail of the vectorised range, at any offset from 16-byte alignment) does
    base = torch.randn(n + 8, device="cuda")
    buf = base[off:off + n]
    tdm.scan_nonfinite(buf)
    assert tdm.ctx_sync() == 0
    for pos in sorted({0, n // 2, n - 1}):
        for bad in (float("nan"), float("inf"), float("-inf")):
            buf[pos] = bad
            tdm.scan_nonfinite(buf)
            assert tdm.ctx_sync() & tdm.FLAG_NONFINITE, (pos, bad)
            buf[pos] = 1.0
    base[off + n] = float("nan")            # just past the end: not scanned
    tdm.scan_nonfinite(buf)
    assert tdm.ctx_sync() == 0


@pytest.mark.parametrize("C,T,B", [(0, 3, 4), (2, 3, 0)])
def test_empty_inputs_write_nothing(tdm, C, T, B):
    # no maps: every entry point returns without touching its (guard-only) outputs
    t = tdm.Tiling(C=C, T=T, B=B, overlap=12, sync_every=1)
    sch = tdm.Schedule(10)
    x0 = torch.zeros(max(C, 1) * T * 4096, device="cuda")
    band = Guarded(0)
    tdm.init_noise(band.t, t, 1)
    tdm.eps_standin(sch, 3, band.t, x0, 0.1, tdm.STREAM_EPS_C, 1, t, band.t)
    tdm.ddim_step(sch, 3, band.t, band.t, band.t, 1.0, 1, t)
    tdm.ddim_run(sch, band.t, x0, 1.0, 0.1, 0.3, 1, t)
    tdm.seam_project(band.t, t)
    seams, tiles = Guarded(C * (T - 1)), Guarded(C * T * 2)
    if B == 0 and C > 0:
        with pytest.raises(tdm.TdmError):           # a mean over no samples
            tdm.seam_discrepancy(band.t, t, seams.t)
    else:
        tdm.seam_discrepancy(band.t, t, seams.t)
    tdm.nonoverlap_drift(band.t, band.t, t, tiles.t, None)
    tdm.kabsch_stitch(band.t, t, band.t, band.t)
    tdm.mds_recover(band.t, 0, band.t, band.t)
    tdm.mds_reconstruct(band.t, 0, band.t, band.t, band.t)
    tdm.pairwise_dist(band.t, 0, band.t)
    tdm.refine_smacof(band.t, 0, band.t, 5, band.t)
    tdm.scan_nonfinite(band.t)
    assert tdm.ctx_sync() == 0
    assert band.intact() and seams.intact() and tiles.intact()
