"""Coordinate recovery: classical MDS and distance reconstruction (oracle side,
float64).

ParaChromo (mdpi.com/2079-9292/15/13/2750) converts each final distance map to a
64-bead point cloud by ChromoGen's distance-geometry initialisation (§3.1, §5.5).
Its formula is not on the pages; the reading here is classical (Torgerson) MDS:

  1. symmetrise D <- (D + D^T) / 2
  2. square entrywise, D2 = D * D
  3. double-centre, B = -1/2 J D2 J with J = I - 1 1^T / n
  4. eigen-decompose B, eigenvalues in descending order
  5. X = [v_1 sqrt(max(l_1, 0)), v_2 sqrt(..), v_3 sqrt(..)]   (n x 3)

The eigen-decomposition is a cyclic Jacobi iteration (Golub & Van Loan,
"Matrix Computations", §8.5: the symmetric 2x2 Schur step, swept in the
round-robin ordering of the parallel Jacobi method), run to convergence in
float64.  The refinement that follows the
initialisation in ChromoGen is not on the pages and is not part of this step.
"""
from __future__ import annotations

import numpy as np


def _sym_schur2(app, aqq, apq):
    """(c, s) zeroing the (p, q) entry of symmetric 2x2 blocks (batched)."""
    nz = apq != 0.0
    safe = np.where(nz, apq, 1.0)
    tau = np.where(nz, (aqq - app) / (2.0 * safe), 0.0)
    t = np.where(tau >= 0.0, 1.0, -1.0) / (np.abs(tau) + np.hypot(1.0, tau))
    t = np.where(nz, t, 0.0)
    c = 1.0 / np.hypot(1.0, t)
    return c, t * c


def round_robin_pairs(n: int):
    """The n-1 rounds of the round-robin ordering: in each round the indices
    0..n-1 (n even) are split into n/2 disjoint pairs (p < q), and over the
    n-1 rounds every pair occurs exactly once."""
    if n % 2:
        raise ValueError("n must be even")
    ring = list(range(1, n))
    rounds = []
    for _ in range(n - 1):
        players = [0] + ring
        pairs = [(players[i], players[n - 1 - i]) for i in range(n // 2)]
        pairs = [(min(a, b), max(a, b)) for a, b in pairs]
        rounds.append((np.array([p for p, _ in pairs]), np.array([q for _, q in pairs])))
        ring = ring[-1:] + ring[:-1]
    return rounds


def jacobi_eigh(A: np.ndarray, tol: float = 1e-12, max_sweeps: int = 60):
    """Eigenvalues and eigenvectors of a batch of symmetric matrices ``A[..., n, n]``.

    Cyclic Jacobi in the round-robin (parallel) ordering: within a round the
    rotations act on disjoint index pairs, so they commute and are applied
    together; one sweep is the n-1 rounds.  Sweeps continue until the
    off-diagonal Frobenius norm is below ``tol`` times the matrix norm.
    Returns ``(lam[..., n], V[..., n, n], sweeps)`` with ``A = V diag(lam) V^T``
    (columns of V are eigenvectors), unsorted.
    """
    A = np.array(A, dtype=np.float64, copy=True)
    shape = A.shape
    n = shape[-1]
    A = A.reshape(-1, n, n)
    V = np.broadcast_to(np.eye(n), A.shape).copy()
    fro = np.sqrt((A * A).sum(axis=(1, 2)))
    offmask = ~np.eye(n, dtype=bool)
    rounds = round_robin_pairs(n)
    sweeps = 0
    for sweeps in range(1, max_sweeps + 1):
        for P, Q in rounds:
            c, s = _sym_schur2(A[:, P, P], A[:, Q, Q], A[:, P, Q])
            cc, ss = c[:, None, :], s[:, None, :]
            ap, aq = A[:, :, P], A[:, :, Q]
            A[:, :, P], A[:, :, Q] = cc * ap - ss * aq, ss * ap + cc * aq
            cr, sr = c[:, :, None], s[:, :, None]
            ap, aq = A[:, P, :], A[:, Q, :]
            A[:, P, :], A[:, Q, :] = cr * ap - sr * aq, sr * ap + cr * aq
            vp, vq = V[:, :, P], V[:, :, Q]
            V[:, :, P], V[:, :, Q] = cc * vp - ss * vq, ss * vp + cc * vq
        off = np.sqrt((A * A * offmask).sum(axis=(1, 2)))
        if np.all(off <= tol * np.maximum(fro, np.finfo(float).tiny)):
            break
    lam = np.diagonal(A, axis1=1, axis2=2).copy()
    return lam.reshape(shape[:-1]), V.reshape(shape), sweeps


def double_center(D2: np.ndarray) -> np.ndarray:
    n = D2.shape[-1]
    J = np.eye(n) - np.ones((n, n)) / n
    return -0.5 * (J @ D2 @ J)


def classical_mds(D: np.ndarray, dims: int = 3):
    """Coordinates ``[..., n, dims]`` and all eigenvalues ``[..., n]`` (descending)."""
    D = np.asarray(D, dtype=np.float64)
    D = 0.5 * (D + np.swapaxes(D, -1, -2))
    B = double_center(D * D)
    lam, V, _ = jacobi_eigh(B)
    order = np.argsort(-lam, axis=-1)
    lam = np.take_along_axis(lam, order, axis=-1)
    V = np.take_along_axis(V, order[..., None, :], axis=-1)
    X = V[..., :dims] * np.sqrt(np.maximum(lam[..., None, :dims], 0.0))
    return X, lam


def pairwise_distances(X: np.ndarray) -> np.ndarray:
    """D_ij = ||x_i - x_j||_2 for coordinates ``X[..., n, d]``."""
    X = np.asarray(X, dtype=np.float64)
    d = X[..., :, None, :] - X[..., None, :, :]
    return np.sqrt((d * d).sum(axis=-1))
