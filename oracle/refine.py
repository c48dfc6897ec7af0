"""Coordinate refinement after the distance-geometry initialisation (oracle
side, float64).

ParaChromo (mdpi.com/2079-9292/15/13/2750), §3.1: a final distance map is
converted to a point cloud by distance-geometry initialisation followed by
coordinate refinement.  The refinement is not specified on the pages; the
reading here is stress minimisation by SMACOF (de Leeuw 1977; Borg & Groenen,
"Modern Multidimensional Scaling", ch. 8): with the raw stress

    sigma(X) = sum_{i<j} (||x_i - x_j|| - D_ij)^2,

each iteration applies the Guttman transform

    X <- (1/n) B(X) X,   B_ij = -D_ij / d_ij(X) (i != j, 0 where d_ij = 0),
                         B_ii = -sum_{j != i} B_ij,

which never increases sigma and, for centred X, is the gradient step of size
1/(2n).  D is first symmetrised, D <- (D + D^T)/2, as for the initialisation.
A fixed number of iterations is run.
"""
from __future__ import annotations

import numpy as np


def pairwise(X):
    d = X[..., :, None, :] - X[..., None, :, :]
    return np.sqrt((d * d).sum(axis=-1))


def stress(X, D) -> np.ndarray:
    """Raw stress of coordinates ``X[..., n, d]`` against maps ``D[..., n, n]``."""
    D = 0.5 * (np.asarray(D, dtype=np.float64) + np.swapaxes(D, -1, -2))
    r = pairwise(np.asarray(X, dtype=np.float64)) - D
    return 0.5 * (r * r).sum(axis=(-1, -2))     # each pair counted once


def guttman_transform(X, D) -> np.ndarray:
    X = np.asarray(X, dtype=np.float64)
    n = X.shape[-2]
    d = pairwise(X)
    safe = np.where(d > 0.0, d, 1.0)
    Bm = np.where(d > 0.0, -D / safe, 0.0)
    idx = np.arange(n)
    Bm[..., idx, idx] = 0.0
    Bm[..., idx, idx] = -Bm.sum(axis=-1)
    return Bm @ X / n


def smacof(X0, D, iterations: int):
    """``iterations`` Guttman transforms from ``X0``; returns (X, stress(X))."""
    D = 0.5 * (np.asarray(D, dtype=np.float64) + np.swapaxes(np.asarray(D, dtype=np.float64), -1, -2))
    X = np.asarray(X0, dtype=np.float64)
    for _ in range(iterations):
        X = guttman_transform(X, D)
    return X, stress(X, D)
