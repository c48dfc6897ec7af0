"""Pins of the oracle's reverse run: closed forms of the ideal denoiser,
statistics of the eta > 0 path, and consistency of sharded runs."""
import numpy as np
import pytest

import synth
from oracle import philox, schedule, seam
from oracle.ddim import (cfg_combine, ddim_run, eps_standin, init_noise, sample_ids,
                         stream_noise)


def _c0(s):
    return np.sqrt(1 - s.ab_t[0]) / np.sqrt(s.ab_t[0])


@pytest.mark.parametrize("w,eta,T,S", [(0.0, 0.0, 4, 50), (1.0, 0.0, 3, 20), (0.5, 1.0, 3, 10),
                                       (1.0, 1.0, 1, 25)])
def test_final_map_closed_form(w, eta, T, S):
    # With the ideal denoiser the last step returns x0 - c0 * (noise part of
    # eps at step 0), c0 = sqrt(1 - ab_0) / sqrt(ab_0) = sqrt(b_0 / (1 - b_0)),
    # whatever happened before; the projection then averages the overlaps,
    # which agree in x0.
    s = schedule.Schedule(S=S, eta=eta)
    assert abs(_c0(s) - np.sqrt(1e-4 / (1 - 1e-4))) < 1e-15
    B, s_c, s_u, seed = 3, 0.1, 0.3, 42
    x0 = synth.chain_x0(2, 2, T).astype(np.float64)
    got = ddim_run(x0, s, w, s_c, s_u, seed, np.arange(B), B)
    g = sample_ids(2, T, np.arange(B), B)
    noise = (1 + w) * s_c * stream_noise(seed, philox.TAG_EPS_C, 0, g)
    if w != 0:
        noise = noise - w * s_u * stream_noise(seed, philox.TAG_EPS_U, 0, g)
    ref = x0[:, :, None] - _c0(s) * noise
    if T > 1:
        ref = seam.seam_project(ref)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_noise_free_trajectory_closed_form():
    # s_c = 0, eta = 0: eps is the ideal one, and every state after the first
    # step is sqrt(ab) x0 + sqrt(1 - ab) P(eps_T), eps_T the noise of x_T.
    S, T, B, seed = 20, 3, 2, 3
    s = schedule.Schedule(S=S)
    x0 = synth.chain_x0(1, 1, T).astype(np.float64)
    final, traj = ddim_run(x0, s, 0.0, 0.0, 0.0, seed, np.arange(B), B, return_trajectory=True)
    g = sample_ids(1, T, np.arange(B), B)
    xT = init_noise(seed, g)
    eps_T = (xT - np.sqrt(s.ab_t[-1]) * x0[:, :, None]) / np.sqrt(1 - s.ab_t[-1])
    p_eps = seam.seam_project(eps_T)
    for n_done, state in enumerate(traj, start=1):
        i = S - n_done
        ab = s.ab_p[i]
        ref = np.sqrt(ab) * x0[:, :, None] + np.sqrt(1 - ab) * p_eps
        np.testing.assert_allclose(state, ref, rtol=0, atol=1e-11)
    np.testing.assert_allclose(final, np.broadcast_to(x0[:, :, None], final.shape), atol=1e-12)


def test_eta_one_keeps_unit_variance_and_step_correlation():
    # With the ideal denoiser the normalised residual e_t = (x_t - sqrt(ab_t) x0)
    # / sqrt(1 - ab_t) obeys e_p = a e_t + b z with a^2 + b^2 = 1,
    # a = sqrt(1 - ab_p - sigma^2) / sqrt(1 - ab_p): unit variance is kept and
    # consecutive residuals correlate by a.
    S, B = 10, 64
    s = schedule.Schedule(S=S, eta=1.0)
    x0 = synth.region_x0(0, [0]).astype(np.float64)   # [1][1][64][64]
    _, traj = ddim_run(x0, s, 0.0, 0.0, 0.0, 11, np.arange(B), B, sync_every=0,
                       return_trajectory=True)
    iu = np.triu_indices(64)
    res = []
    for n_done, state in enumerate(traj[:-1], start=1):
        i = S - n_done
        e = (state - np.sqrt(s.ab_p[i]) * x0[:, :, None]) / np.sqrt(1 - s.ab_p[i])
        res.append(e[..., iu[0], iu[1]].ravel())
    n = res[0].size
    for k, e in enumerate(res):
        assert abs(e.var() - 1.0) < 6 * np.sqrt(2.0 / n), (k, e.var())
    for k in range(1, len(res)):
        i = S - k - 1                     # the step from residual k-1 to k
        a = np.sqrt(1 - s.ab_p[i] - s.sigma[i] ** 2) / np.sqrt(1 - s.ab_p[i])
        r = np.corrcoef(res[k - 1], res[k])[0, 1]
        assert abs(r - a) < 6.0 / np.sqrt(n), (k, r, a)


def test_cfg_combination():
    rng = np.random.default_rng(0)
    ec, eu = rng.standard_normal((2, 100))
    np.testing.assert_array_equal(cfg_combine(ec, eu, 0.0), ec)
    np.testing.assert_allclose(cfg_combine(ec, eu, 1.0), 2 * ec - eu, rtol=1e-15)
    # eps_standin with s = 0 is the ideal eps: x_t built from x0 and e gives e back
    x0, e = rng.standard_normal((2, 100))
    ab = 0.3
    np.testing.assert_allclose(eps_standin(np.sqrt(ab) * x0 + np.sqrt(1 - ab) * e, x0, ab, 0.0, 0.0),
                               e, rtol=1e-13, atol=1e-13)


def test_sharded_run_equals_full_run():
    # samples split in two shards (with their global indices) reproduce the
    # corresponding samples of the unsplit run exactly
    s = schedule.Schedule(S=5)
    x0 = synth.chain_x0(4, 1, 3).astype(np.float64)
    full = ddim_run(x0, s, 1.0, 0.1, 0.3, 9, np.arange(6), 6)
    a = ddim_run(x0, s, 1.0, 0.1, 0.3, 9, np.arange(0, 4), 6)
    b = ddim_run(x0, s, 1.0, 0.1, 0.3, 9, np.arange(4, 6), 6)
    np.testing.assert_array_equal(np.concatenate([a, b], axis=2), full)


def test_states_stay_symmetric_and_given_start_is_folded():
    s = schedule.Schedule(S=4, eta=1.0)
    x0 = synth.chain_x0(5, 1, 2).astype(np.float64)
    xT = synth.gaussian_maps(1, 4, symmetric=False).astype(np.float64).reshape(1, 2, 2, 64, 64)
    out = ddim_run(x0, s, 1.0, 0.1, 0.3, 1, np.arange(2), 2, x_T=xT)
    np.testing.assert_array_equal(out, np.swapaxes(out, -1, -2))
    sym = np.triu(xT) + np.swapaxes(np.triu(xT, 1), -1, -2)
    np.testing.assert_array_equal(out, ddim_run(x0, s, 1.0, 0.1, 0.3, 1, np.arange(2), 2, x_T=sym))
