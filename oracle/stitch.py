"""Kabsch stitching of per-tile coordinates into one chain (oracle side,
float64).

ParaChromo (mdpi.com/2079-9292/15/13/2750), §4.3.2 (last paragraph) and §5.5
with Fig. 4: the coordinates of each tile come from the coordinate-recovery
step separately; adjacent tiles are stitched by Kabsch alignment on their
12-bead overlap, and the per-seam Kabsch residual after stitching is reported.
Readings (the pages give no formulas):

  * tile k+1 is aligned onto tile k by the rigid map x -> R x + t minimising
    sum_i |R q_i + t - p_i|^2 over the overlap beads, p_i = tile k's beads
    [s, 64), q_i = tile k+1's beads [0, o); R may be improper (det -1),
    because recovered coordinates are defined only up to reflection;
  * the maps compose along the chain, so every tile lands in tile 0's frame;
  * an overlap bead takes the mean of its two aligned copies;
  * the residual of a seam is the RMSD over its o beads after alignment.

The rotation is the orthogonal polar factor of the cross-covariance (Kabsch /
orthogonal Procrustes), computed with numpy's SVD.
"""
from __future__ import annotations

import numpy as np


def procrustes(P: np.ndarray, Q: np.ndarray):
    """(R, t, rmsd) with R orthogonal minimising |R Q_i + t - P_i| over rows."""
    P = np.asarray(P, dtype=np.float64)
    Q = np.asarray(Q, dtype=np.float64)
    pc, qc = P.mean(axis=0), Q.mean(axis=0)
    M = (P - pc).T @ (Q - qc)                 # sum_i p_i q_i^T
    U, _, Vt = np.linalg.svd(M)
    R = U @ Vt
    t = pc - R @ qc
    res = (Q @ R.T + t) - P
    return R, t, float(np.sqrt((res * res).sum(axis=1).mean()))


def stitch(coords: np.ndarray, overlap: int = 12):
    """coords ``[C][T][B][n][3]`` -> (chains ``[C][B][L][3]``, residuals
    ``[C][B][T-1]``), L = n + (T-1)(n - overlap)."""
    X = np.asarray(coords, dtype=np.float64)
    C, T, B, n, _ = X.shape
    s = n - overlap
    L = n + (T - 1) * s
    chains = np.zeros((C, B, L, 3))
    resid = np.zeros((C, B, max(T - 1, 0)))
    for c in range(C):
        for b in range(B):
            G_R, G_t = np.eye(3), np.zeros(3)          # tile k -> tile 0 frame
            placed = []
            for k in range(T):
                placed.append(X[c, k, b] @ G_R.T + G_t)
                if k < T - 1:
                    R, t, rmsd = procrustes(X[c, k, b, s:], X[c, k + 1, b, :overlap])
                    resid[c, b, k] = rmsd
                    G_t = G_R @ t + G_t
                    G_R = G_R @ R
            for k in range(T):
                lo = k * s
                if k == 0:
                    chains[c, b, 0:n] = placed[0]
                else:
                    # overlap beads: mean of tile k-1's and tile k's copies
                    chains[c, b, lo:lo + overlap] = 0.5 * (chains[c, b, lo:lo + overlap] + placed[k][:overlap])
                    chains[c, b, lo + overlap:lo + n] = placed[k][overlap:]
    return chains, resid
