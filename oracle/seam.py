"""Overlap-consistency projection and seam discrepancy (oracle side, float64).

ParaChromo (mdpi.com/2079-9292/15/13/2750), §4.3.2 and Algorithm 1: for every
adjacent pair of regions, the right-overlap subblock of the left region and the
left-overlap subblock of the right region describe the same bead pairs (§3.2:
the lower-right block of the left region and the upper-left block of the right
region); both are replaced in place by their elementwise mean.  The same sample
index b across regions is one joint tiled sample (§4.3.2), so only maps with
equal b are coupled.  The Algorithm 1 body is empty on the page; its prose
steps are unfold -> average -> refold, and the unfold/refold (the origami
transform) is the identity here because the state kept is the unfolded
symmetric map.

Seam discrepancy, §5.5 Eq. (6) (body lost on the page; read from its prose):
for the seam between tiles k and k+1, the mean over the o x o overlap entries
of |mean_b D_k[s+i, s+j] - mean_b D_{k+1}[i, j]|, where s = n - o.

Maps are laid out ``[C][T][B][n][n]``.
"""
from __future__ import annotations

import numpy as np


def unique_beads(T: int, n: int = 64, overlap: int = 12) -> int:
    """Beads covered by T tiles of n beads with adjacent tiles sharing ``overlap``."""
    return T * n - (T - 1) * overlap


def n_seams(T: int) -> int:
    return max(T - 1, 0)


def right_block(X: np.ndarray, overlap: int) -> np.ndarray:
    n = X.shape[-1]
    return X[..., n - overlap:, n - overlap:]


def left_block(X: np.ndarray, overlap: int) -> np.ndarray:
    return X[..., :overlap, :overlap]


def seam_project(X: np.ndarray, overlap: int = 12) -> np.ndarray:
    """Return the projected copy of ``X[C][T][B][n][n]``."""
    Y = np.array(X, dtype=np.float64, copy=True)
    T = Y.shape[1]
    n = Y.shape[-1]
    s = n - overlap
    for k in range(T - 1):
        a = Y[:, k, :, s:, s:]
        b = Y[:, k + 1, :, :overlap, :overlap]
        m = (a + b) / 2.0
        Y[:, k, :, s:, s:] = m
        Y[:, k + 1, :, :overlap, :overlap] = m
    return Y


def seam_discrepancy(X: np.ndarray, overlap: int = 12) -> np.ndarray:
    """Eq. (6) per chain and seam: ``[C][T-1]`` float64."""
    X = np.asarray(X, dtype=np.float64)
    C, T = X.shape[0], X.shape[1]
    n = X.shape[-1]
    s = n - overlap
    out = np.zeros((C, max(T - 1, 0)))
    for c in range(C):
        for k in range(T - 1):
            mean_right = X[c, k, :, s:, s:].mean(axis=0)
            mean_left = X[c, k + 1, :, :overlap, :overlap].mean(axis=0)
            out[c, k] = np.abs(mean_right - mean_left).mean()
    return out


def overlap_difference_sums(X: np.ndarray, overlap: int = 12) -> np.ndarray:
    """Per chain and seam, the sum over samples of (right block - left block):
    ``[C][T-1][o][o]``.  Eq. (6) of a set of samples split into shards is the
    mean of |sum over all shards / B| over the overlap entries."""
    X = np.asarray(X, dtype=np.float64)
    n = X.shape[-1]
    s = n - overlap
    return (X[:, :-1, :, s:, s:] - X[:, 1:, :, :overlap, :overlap]).sum(axis=2)


def discrepancy_from_sums(sums: np.ndarray, B_total: int) -> np.ndarray:
    return np.abs(sums / B_total).mean(axis=(-1, -2))
