"""Stand-in denoiser, classifier-free guidance and the DDIM reverse run
(oracle side, float64).

The trained ChromoGen U-Net of ParaChromo (mdpi.com/2079-9292/15/13/2750, §3.1)
is replaced by a seeded stand-in: the ideal denoiser toward a known x0 plus
Philox noise,

    eps_ideal = (x_t - sqrt(ab_t) x0) / sqrt(1 - ab_t)
    eps_c     = eps_ideal + s_c z_c        (conditional stream)
    eps_u     = eps_ideal + s_u z_u        (unconditional stream)

combined by classifier-free guidance (the pages' ref. [15], Ho & Salimans) as
eps = (1 + w) eps_c - w eps_u; at w = 0 the unconditional stream is not drawn.

The DDIM update (Song et al., the pages' ref. [7]) is written in its three
terms: the predicted x0, the direction pointing to x_t, and the random noise.
The overlap projection (§4.3.2) follows the update of every K-th step, counting
steps done, including the last one.

Maps are ``[C][T][B][n][n]``; x0 is ``[C][T][n][n]`` shared by the B samples
(§3.3: samples of one condition differ only through their noise).  Sample b of
tile k of chain c has noise id

    g = sample_id_base + (c*T + k) * B_total + b_index

where ``b_index`` is the sample's index among all B_total samples of the run.
"""
from __future__ import annotations

import numpy as np

from .philox import (TAG_EPS_C, TAG_EPS_U, TAG_ETA, TAG_INIT, symmetric_normal)
from .schedule import Schedule
from .seam import seam_project


def eps_ideal(x_t, x0, ab_t):
    return (x_t - np.sqrt(ab_t) * x0) / np.sqrt(1.0 - ab_t)


def eps_standin(x_t, x0, ab_t, s, z):
    return eps_ideal(x_t, x0, ab_t) + s * z


def cfg_combine(eps_c, eps_u, w):
    return (1.0 + w) * eps_c - w * eps_u


def predict_x0(x_t, eps, ab_t):
    return (x_t - np.sqrt(1.0 - ab_t) * eps) / np.sqrt(ab_t)


def ddim_update(x_t, eps, ab_t, ab_p, sigma, z=None):
    """x_{tau_{i-1}} from x_{tau_i} (Song et al., eq. 12)."""
    x0_hat = predict_x0(x_t, eps, ab_t)
    direction = np.sqrt(max(1.0 - ab_p - sigma * sigma, 0.0)) * eps
    out = np.sqrt(ab_p) * x0_hat + direction
    if sigma != 0.0:
        out = out + sigma * z
    return out


def ddpm_ancestral_step(x_t, eps, t, betas, ab, z):
    """One DDPM ancestral step t -> t-1 with the posterior variance beta-tilde
    (Ho et al. 2020); written independently of :func:`ddim_update`."""
    ab_t = ab[t]
    ab_prev = ab[t - 1] if t > 0 else 1.0
    alpha_t = 1.0 - betas[t]
    x0_hat = (x_t - np.sqrt(1.0 - ab_t) * eps) / np.sqrt(ab_t)
    mean = (np.sqrt(ab_prev) * betas[t] / (1.0 - ab_t)) * x0_hat \
        + (np.sqrt(alpha_t) * (1.0 - ab_prev) / (1.0 - ab_t)) * x_t
    var = (1.0 - ab_prev) / (1.0 - ab_t) * betas[t]
    return mean + np.sqrt(var) * z


def sample_ids(C: int, T: int, b_index, B_total: int, sample_id_base: int = 0) -> np.ndarray:
    """Noise ids ``[C][T][len(b_index)]`` (uint64)."""
    b_index = np.asarray(b_index, dtype=np.int64)
    c = np.arange(C, dtype=np.int64)[:, None, None]
    k = np.arange(T, dtype=np.int64)[None, :, None]
    return (sample_id_base + (c * T + k) * B_total + b_index[None, None, :]).astype(np.uint64)


def fold(x):
    """The folded state of a map: its upper triangle (i <= j), mirrored back to
    a full symmetric map.  The fused run keeps only this triangle."""
    return np.triu(x) + np.swapaxes(np.triu(x, 1), -1, -2)


def init_noise(seed: int, g) -> np.ndarray:
    """x_T: the symmetric N(0,1) field of the INIT stream (step word 0)."""
    g = np.asarray(g, dtype=np.uint64)
    return symmetric_normal(seed, TAG_INIT, 0, g.reshape(-1)).reshape(g.shape + (64, 64))


def stream_noise(seed: int, tag: int, step: int, g) -> np.ndarray:
    g = np.asarray(g, dtype=np.uint64)
    return symmetric_normal(seed, tag, step, g.reshape(-1)).reshape(g.shape + (64, 64))


def ddim_run(x0, sched: Schedule, w: float, s_c: float, s_u: float, seed: int,
             b_index, B_total: int, overlap: int = 12, sync_every: int = 1,
             sample_id_base: int = 0, x_T=None, return_trajectory: bool = False):
    """The whole reverse run for the samples ``b_index`` of every chain and tile.

    ``x0``: ``[C][T][n][n]``.  ``x_T``: optional ``[C][T][len(b_index)][n][n]``
    starting state (its folded triangle is used); default: the INIT noise.
    Returns the final maps ``[C][T][Bs][n][n]`` (and the list of states after
    every step when ``return_trajectory``).
    """
    x0 = np.asarray(x0, dtype=np.float64)
    C, T = x0.shape[0], x0.shape[1]
    g = sample_ids(C, T, b_index, B_total, sample_id_base)
    x0b = x0[:, :, None, :, :]
    if x_T is None:
        x = init_noise(seed, g)
    else:
        x = fold(np.asarray(x_T, dtype=np.float64))
    traj = []
    S = sched.S
    for i in reversed(range(S)):
        ab_t, ab_p, sigma = sched.ab_t[i], sched.ab_p[i], sched.sigma[i]
        eps = eps_standin(x, x0b, ab_t, s_c, stream_noise(seed, TAG_EPS_C, i, g))
        if w != 0.0:
            eps_u = eps_standin(x, x0b, ab_t, s_u, stream_noise(seed, TAG_EPS_U, i, g))
            eps = cfg_combine(eps, eps_u, w)
        z = stream_noise(seed, TAG_ETA, i, g) if sched.eta > 0.0 else None
        x = ddim_update(x, eps, ab_t, ab_p, sigma, z)
        if T > 1 and sync_every > 0 and (S - i) % sync_every == 0:
            x = seam_project(x, overlap)
        if return_trajectory:
            traj.append(x.copy())
    return (x, traj) if return_trajectory else x
