"""Noise schedule and DDIM step coefficients (oracle side, float64).

ParaChromo (mdpi.com/2079-9292/15/13/2750) runs the trained denoiser with DDIM
at a reduced step count (§4.1, §5.1.1, §5.4.3) and names a cosine-beta schedule
(§4.3.2) without its constants; the workloads here use a linear beta schedule
1e-4 .. 0.02 over 1000 training steps, and an arbitrary alphas-bar table may be
passed instead.  The DDIM update itself is not printed on the pages; it is the
one of Song, Meng, Ermon, "Denoising Diffusion Implicit Models" (the pages'
ref. [7]), read as:

  * timesteps tau_i = i * (T_train / S), i = 0 .. S-1, the reverse loop runs
    i = S-1 .. 0, and alphas_bar before tau_0 is 1 (the last step returns the
    predicted x0);
  * sigma_i = eta * sqrt((1 - ab_p) / (1 - ab_t)) * sqrt(1 - ab_t / ab_p)
    with ab_t = alphas_bar[tau_i], ab_p = alphas_bar[tau_{i-1}].
"""
from __future__ import annotations

import numpy as np


def linear_betas(T_train: int = 1000, beta_start: float = 1e-4, beta_end: float = 0.02) -> np.ndarray:
    """beta_t for t = 0 .. T_train-1, evenly spaced from beta_start to beta_end."""
    t = np.arange(T_train, dtype=np.float64)
    return beta_start + (beta_end - beta_start) * t / (T_train - 1)


def alphas_bar(betas: np.ndarray) -> np.ndarray:
    """alphas_bar_t = prod_{s <= t} (1 - beta_s)."""
    out = np.empty_like(betas)
    acc = 1.0
    for t, b in enumerate(betas):
        acc *= (1.0 - b)
        out[t] = acc
    return out


def cosine_alphas_bar(T_train: int = 1000, s: float = 0.008, max_beta: float = 0.999) -> np.ndarray:
    """The cosine schedule of Nichol & Dhariwal, "Improved Denoising Diffusion
    Probabilistic Models" (ICML 2021, section 3.2): alphas_bar(t) = f(t) / f(0)
    with f(t) = cos^2(((t / T) + s) / (1 + s) * pi / 2), beta clipped at
    max_beta.  Entry k of the table is timestep t = k + 1 (entry 0 is the first
    noising step).  ParaChromo §4.3.2 names a cosine schedule; its constants
    are not on the pages, so the published ones are used."""
    def f(t):
        return np.cos(((t / T_train) + s) / (1.0 + s) * np.pi / 2.0) ** 2

    out = np.empty(T_train)
    acc = 1.0
    for k in range(T_train):
        beta = min(1.0 - f(k + 1.0) / f(float(k)), max_beta)
        acc *= 1.0 - beta
        out[k] = acc
    return out


def ddim_timesteps(T_train: int, S: int) -> np.ndarray:
    if S < 1 or T_train % S != 0:
        raise ValueError("S must divide T_train")
    return np.arange(S, dtype=np.int64) * (T_train // S)


def ddim_table(ab: np.ndarray, S: int, eta: float):
    """Per DDIM step i: (tau_i, ab_t, ab_p, sigma_i) as float64 arrays of length S."""
    T_train = len(ab)
    tau = ddim_timesteps(T_train, S)
    ab_t = ab[tau]
    ab_p = np.empty(S)
    ab_p[0] = 1.0
    ab_p[1:] = ab[tau[:-1]]
    sigma = eta * np.sqrt((1.0 - ab_p) / (1.0 - ab_t)) * np.sqrt(1.0 - ab_t / ab_p)
    return tau, ab_t, ab_p, sigma


class Schedule:
    """The schedule of one sampler configuration."""

    def __init__(self, T_train: int = 1000, beta_start: float = 1e-4, beta_end: float = 0.02,
                 S: int = 50, eta: float = 0.0, alphas_bar_table=None):
        if alphas_bar_table is None:
            self.betas = linear_betas(T_train, beta_start, beta_end)
            self.ab = alphas_bar(self.betas)
        else:
            self.ab = np.asarray(alphas_bar_table, dtype=np.float64)
            prev = np.concatenate([[1.0], self.ab[:-1]])
            self.betas = 1.0 - self.ab / prev
        self.T_train = len(self.ab)
        self.S = S
        self.eta = eta
        self.tau, self.ab_t, self.ab_p, self.sigma = ddim_table(self.ab, S, eta)
