"""Pins of the oracle's schedule and DDIM coefficients."""
import numpy as np
import pytest

from oracle import schedule
from oracle.ddim import ddim_update, ddpm_ancestral_step


def test_linear_betas_endpoints():
    b = schedule.linear_betas(1000, 1e-4, 0.02)
    assert b[0] == 1e-4 and abs(b[-1] - 0.02) < 1e-17 and len(b) == 1000
    assert np.allclose(np.diff(b), (0.02 - 1e-4) / 999, rtol=0, atol=1e-17)


def test_alphas_bar_against_log_series():
    # log prod(1 - b) = -sum b - sum b^2 / 2 - R with 0 <= R <= sum b^3 (b <= 0.02)
    b = schedule.linear_betas()
    ab = schedule.alphas_bar(b)
    assert ab[0] == 1.0 - 1e-4
    lo = -b.sum() - (b ** 2).sum() / 2 - (b ** 3).sum()
    hi = -b.sum() - (b ** 2).sum() / 2
    assert lo <= np.log(ab[-1]) <= hi
    assert 4.0e-5 < ab[-1] < 4.1e-5
    assert np.all(np.diff(ab) < 0)


def test_timesteps():
    np.testing.assert_array_equal(schedule.ddim_timesteps(1000, 50), np.arange(0, 1000, 20))
    np.testing.assert_array_equal(schedule.ddim_timesteps(1000, 1000), np.arange(1000))
    with pytest.raises(ValueError):
        schedule.ddim_timesteps(1000, 30)


def test_last_step_has_alpha_prev_one_and_no_noise():
    for eta in (0.0, 0.5, 1.0):
        s = schedule.Schedule(S=50, eta=eta)
        assert s.ab_p[0] == 1.0 and s.sigma[0] == 0.0
        assert s.tau[0] == 0 and s.tau[-1] == 980
        np.testing.assert_array_equal(s.ab_p[1:], s.ab_t[:-1])


def test_eta_one_full_length_is_posterior_variance():
    # DDIM sigma at eta=1 with every timestep equals the DDPM posterior std
    s = schedule.Schedule(S=1000, eta=1.0)
    t = np.arange(1, 1000)
    beta_tilde = (1.0 - s.ab[t - 1]) / (1.0 - s.ab[t]) * s.betas[t]
    np.testing.assert_allclose(s.sigma[1:] ** 2, beta_tilde, rtol=1e-12)


def test_ddim_eta_one_equals_ddpm_ancestral_step():
    s = schedule.Schedule(S=1000, eta=1.0)
    rng = np.random.default_rng(5)
    for t in (0, 1, 2, 17, 500, 998, 999):
        x, e, z = rng.standard_normal((3, 64))
        a = ddim_update(x, e, s.ab_t[t], s.ab_p[t], s.sigma[t], z)
        b = ddpm_ancestral_step(x, e, t, s.betas, s.ab, z)
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("eta", [0.0, 1.0])
def test_ddim_preserves_forward_marginal_form(eta):
    # with the exact noise eps of x_t = sqrt(ab_t) x0 + sqrt(1-ab_t) eps and
    # no fresh noise, one step lands on sqrt(ab_p) x0 + (direction) eps
    s = schedule.Schedule(S=50, eta=eta)
    rng = np.random.default_rng(9)
    x0, e = rng.standard_normal((2, 256))
    for i in range(50):
        xt = np.sqrt(s.ab_t[i]) * x0 + np.sqrt(1 - s.ab_t[i]) * e
        out = ddim_update(xt, e, s.ab_t[i], s.ab_p[i], s.sigma[i], np.zeros_like(e))
        ref = np.sqrt(s.ab_p[i]) * x0 + np.sqrt(1 - s.ab_p[i] - s.sigma[i] ** 2) * e
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_cosine_schedule_closed_forms():
    # with s = 0 and no beta reaching the clip, alphas_bar(t) telescopes to
    # cos^2(pi t / 2T): 1/2 at t = T/2 and 3/4 at t = T/3 (entry t - 1)
    ab = schedule.cosine_alphas_bar(1200, s=0.0)
    assert ab[600 - 1] == pytest.approx(0.5, rel=1e-12)
    assert ab[400 - 1] == pytest.approx(0.75, rel=1e-12)
    assert ab[0] == pytest.approx(np.cos(np.pi / 2400) ** 2, rel=1e-14)


def test_cosine_schedule_clip_and_order():
    ab = schedule.cosine_alphas_bar(1000)
    assert np.all(np.diff(ab) < 0) and ab[0] < 1.0 and ab[-1] > 0.0
    betas = 1.0 - ab / np.concatenate([[1.0], ab[:-1]])
    assert betas[-1] == pytest.approx(0.999, rel=1e-12)     # f(T) = 0 is clipped
    assert betas.max() <= 0.999 + 1e-12
    # the offset s keeps the first beta small: 1 - f(1)/f(0) for s = 0.008
    f = lambda t: np.cos((t / 1000 + 0.008) / 1.008 * np.pi / 2) ** 2
    assert betas[0] == pytest.approx(1 - f(1) / f(0), rel=1e-12)
    # a schedule built from the table accepts it as given
    sch = schedule.Schedule(S=50, alphas_bar_table=ab)
    np.testing.assert_allclose(sch.ab_t, ab[::20])
