"""Pins of the oracle's non-overlap drift (ParaChromo §5.7, Table 8)."""
import numpy as np
import pytest

import synth
from oracle import ddim, drift, schedule, seam


def _maps(seed, C, T, B):
    return synth.gaussian_maps(seed, C * T * B).astype(np.float64).reshape(C, T, B, 64, 64)


@pytest.mark.parametrize("T,k,count", [(1, 0, 4096), (2, 0, 4096 - 144), (2, 1, 4096 - 144),
                                       (5, 0, 4096 - 144), (5, 2, 4096 - 288), (5, 4, 4096 - 144)])
def test_mask_counts(T, k, count):
    # tiles at the chain ends have one overlap block, interior tiles two, and
    # a lone tile none
    assert drift.nonoverlap_mask(T, k).sum() == count


def test_mask_blocks_are_the_seam_blocks():
    # the masked entries are exactly those the projection writes
    T, o = 4, 12
    X = _maps(1, 1, T, 1)
    P = seam.seam_project(X, o)
    for k in range(T):
        changed = P[0, k, 0] != X[0, k, 0]
        assert not np.any(changed & drift.nonoverlap_mask(T, k, o))


def test_uniform_relative_change_gives_its_size():
    # S = V (1 + eps) on positive V: drift = eps exactly
    V = np.abs(_maps(2, 2, 3, 4)) + 0.5
    for eps in (0.0, 0.01, 0.3):
        r = drift.relative_drift(V * (1 + eps), V)
        np.testing.assert_allclose(r, eps, rtol=1e-12, atol=1e-15)


def test_changes_inside_the_overlap_blocks_do_not_count():
    V = _maps(3, 1, 3, 2)
    S = V.copy()
    S[0, 0, :, 52:, 52:] += 7.0
    S[0, 1, :, :12, :12] -= 3.0
    S[0, 1, :, 52:, 52:] *= 2.0
    S[0, 2, :, :12, :12] = 0.0
    assert np.all(drift.drift_sums(S, V)[..., 0] == 0.0)


def test_one_entry_change():
    V = _maps(4, 1, 3, 2)
    S = V.copy()
    S[0, 1, 1, 30, 5] += 0.25
    s = drift.drift_sums(S, V)
    assert s[0, 1, 0] == pytest.approx(0.25, abs=1e-15)
    assert s[0, 0, 0] == 0.0 and s[0, 2, 0] == 0.0


def test_elementwise_denoiser_never_drifts():
    # with the ideal-denoiser stand-in every entry evolves on its own, so the
    # projection never reaches a non-overlap entry: synchronised and independent
    # runs of the same seeds agree there at every step
    x0 = synth.chain_x0(0, 1, 3)
    sch = schedule.Schedule(S=20, eta=1.0)
    sync = ddim.ddim_run(x0, sch, 0.0, 0.1, 0.0, 5, np.arange(3), 3, sync_every=1)
    free = ddim.ddim_run(x0, sch, 0.0, 0.1, 0.0, 5, np.arange(3), 3, sync_every=0)
    assert np.all(drift.drift_sums(sync, free)[..., 0] == 0.0)
    assert np.all(seam.seam_discrepancy(sync) == 0.0) and np.all(seam.seam_discrepancy(free) > 0.0)
