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


def test_constant_shift_on_tiles_of_different_scale():
    # tiles of value 1, 2 and 4 shifted by 0.1: the drift is a ratio of sums,
    # 0.1 (3952 + 3808 + 3952) / (3952 + 2 * 3808 + 4 * 3952) = 0.0427820...,
    # not the mean of the element ratios (0.0584...)
    V = np.ones((1, 3, 2, 64, 64)) * np.array([1.0, 2.0, 4.0])[None, :, None, None, None]
    r = drift.relative_drift(V + 0.1, V)
    assert r[0] == pytest.approx(0.1 * 11712 / 27376, rel=1e-12)


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


_PINS = [lambda: [test_mask_counts(T, k, c) for T, k, c in ((1, 0, 4096), (2, 0, 3952), (5, 2, 3808), (5, 4, 3952))],
         test_mask_blocks_are_the_seam_blocks, test_uniform_relative_change_gives_its_size,
         test_constant_shift_on_tiles_of_different_scale,
         test_changes_inside_the_overlap_blocks_do_not_count, test_one_entry_change]


@pytest.mark.parametrize("mistake", ["right_block_only", "swapped_blocks", "den_of_s", "mean_of_ratios",
                                     "whole_rows"])
def test_pins_catch_planted_mistakes(mistake, monkeypatch):
    # plant a plausible mistake in the oracle; at least one pin must fail
    orig_mask, orig_sums = drift.nonoverlap_mask, drift.drift_sums

    def bad_mask(T, k, overlap=12, n=64):
        m = np.ones((n, n), dtype=bool)
        if mistake == "right_block_only":
            if k < T - 1:
                m[n - overlap:, n - overlap:] = False
        elif mistake == "swapped_blocks":
            if k < T - 1:
                m[:overlap, :overlap] = False
            if k > 0:
                m[n - overlap:, n - overlap:] = False
        elif mistake == "whole_rows":
            if k > 0:
                m[:overlap, :] = False
            if k < T - 1:
                m[n - overlap:, :] = False
        return m

    def bad_sums(S, V, overlap=12):
        out = orig_sums(S, V, overlap)
        if mistake == "den_of_s":
            out[..., 1] = orig_sums(V, S, overlap)[..., 1]
        return out

    def bad_ratio(S, V, overlap=12):
        with np.errstate(invalid="ignore", divide="ignore"):
            r = np.abs(np.asarray(S, float) - V) / np.abs(np.asarray(V, float))
        C, T = S.shape[:2]
        return np.array([np.nanmean(np.concatenate([r[c, k][..., orig_mask(T, k, overlap)].ravel()
                                                    for k in range(T)])) for c in range(C)])

    if mistake in ("right_block_only", "swapped_blocks", "whole_rows"):
        monkeypatch.setattr(drift, "nonoverlap_mask", bad_mask)
    elif mistake == "den_of_s":
        monkeypatch.setattr(drift, "drift_sums", bad_sums)
    else:
        monkeypatch.setattr(drift, "relative_drift", bad_ratio)
    failed = 0
    for pin in _PINS:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, f"no pin caught {mistake}"
