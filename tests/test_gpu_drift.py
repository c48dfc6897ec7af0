"""GPU parity of the non-overlap drift (ParaChromo §5.7, Table 8) against the
float64 oracle, and the synchronisation-frequency sweep on the sampler."""
import numpy as np
import pytest

import synth
from oracle import drift as odrift, seam as oseam
from tests.gpu_util import TOL_SEAM, dev, host, needs_gpu, torch

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


def _pair(seed, C, T, B, scale=0.05):
    V = synth.gaussian_maps(seed, C * T * B).reshape(C, T, B, 64, 64)
    g = np.random.default_rng([seed, 0xD1F7])
    S = (V + scale * g.standard_normal(V.shape)).astype(np.float32)
    return S, V


def _gpu(tdm, S, V, t, want_ratio=True):
    sums = torch.empty(t.C * t.T * 2, device="cuda")
    ratio = torch.empty(t.C, device="cuda") if want_ratio else None
    tdm.nonoverlap_drift(dev(S).reshape(-1), dev(V).reshape(-1), t, sums, ratio)
    torch.cuda.synchronize()
    return host(sums).reshape(t.C, t.T, 2), (host(ratio) if want_ratio else None)


@pytest.mark.parametrize("C,T,B,o", [(1, 1, 3, 12), (2, 2, 5, 12), (3, 5, 7, 8), (1, 4, 1, 32),
                                     (2, 3, 4, 1), (1, 32, 100, 12), (40, 16, 2, 12)])
def test_drift_matches_oracle(tdm, C, T, B, o):
    # (1, 32, 100): few tiles, samples split over CTAs; (40, 16, 2): one CTA per tile
    S, V = _pair(C * 100 + T, C, T, B)
    t = tdm.Tiling(C=C, T=T, B=B, overlap=o)
    got, ratio = _gpu(tdm, S, V, t)
    want = odrift.drift_sums(S, V, o)
    np.testing.assert_allclose(got, want, rtol=TOL_SEAM)
    np.testing.assert_allclose(ratio, odrift.relative_drift(S, V, o), rtol=TOL_SEAM)


def test_sums_without_ratio(tdm):
    for C, T, B in ((1, 3, 50), (700, 1, 1)):
        S, V = _pair(7 + C, C, T, B)
        t = tdm.Tiling(C=C, T=T, B=B)
        got, _ = _gpu(tdm, S, V, t, want_ratio=False)
        np.testing.assert_allclose(got, odrift.drift_sums(S, V), rtol=TOL_SEAM)


def test_identical_maps_and_blocks_only_changes(tdm):
    S, V = _pair(11, 2, 4, 3)
    t = tdm.Tiling(C=2, T=4, B=3)
    got, ratio = _gpu(tdm, V, V, t)
    assert np.all(got[..., 0] == 0.0) and np.all(ratio == 0.0)
    W = V.copy()
    W[:, :-1, :, 52:, 52:] += 5.0
    W[:, 1:, :, :12, :12] -= 5.0
    got, _ = _gpu(tdm, W, V, t)
    assert np.all(got[..., 0] == 0.0)


@pytest.mark.parametrize("K", [1, 10, 100, 7])
def test_sync_interval_sweep_ddpm(tdm, K):
    # three tiles x 8 samples, the 1000-step DDPM ancestral sampler (DDIM eta 1 at
    # S = T_train), projection every K steps against an independent run of the
    # same seeds: the stand-in denoiser acts entry by entry, so outside the
    # overlap blocks the two runs agree bit for bit; when K divides 1000 the
    # last step is projected and the overlap discrepancy of Eq. (6) is 0
    T, B = 3, 8
    x0 = synth.chain_x0(1, 1, T)
    sch = tdm.Schedule(1000, eta=1.0)
    out = {}
    for k in (K, 0):
        t = tdm.Tiling(C=1, T=T, B=B, overlap=12, sync_every=k)
        maps = torch.empty(T * B * 4096, device="cuda")
        tdm.ddim_run(sch, maps, dev(x0).reshape(-1), 0.0, 0.1, 0.0, 3, t)
        out[k] = maps
    t = tdm.Tiling(C=1, T=T, B=B, overlap=12)
    sums = torch.empty(T * 2, device="cuda")
    ratio = torch.empty(1, device="cuda")
    tdm.nonoverlap_drift(out[K], out[0], t, sums, ratio)
    disc = torch.empty(T - 1, device="cuda")
    tdm.seam_discrepancy(out[K], t, disc)
    torch.cuda.synchronize()
    assert np.all(host(sums).reshape(T, 2)[:, 0] == 0.0) and host(ratio)[0] == 0.0
    free = host(out[0]).reshape(1, T, B, 64, 64)
    assert np.all(oseam.seam_discrepancy(free) > 0.0)
    if 1000 % K == 0:
        assert np.all(host(disc) == 0.0)
    else:
        assert np.all(host(disc) > 0.0)


def test_drift_full_size(tdm):
    # the 32-tile x 1000-sample chain: 32,000 map pairs
    C, T, B = 1, 32, 1000
    S, V = _pair(5, C, T, B, scale=0.01)
    t = tdm.Tiling(C=C, T=T, B=B)
    got, ratio = _gpu(tdm, S, V, t)
    np.testing.assert_allclose(got, odrift.drift_sums(S, V), rtol=TOL_SEAM)
    np.testing.assert_allclose(ratio, odrift.relative_drift(S, V), rtol=TOL_SEAM)
