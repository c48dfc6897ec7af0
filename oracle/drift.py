"""Non-overlap drift of synchronised maps from an unsynchronised run (oracle
side, float64).  Test infrastructure only, like the rest of this package.

ParaChromo (mdpi.com/2079-9292/15/13/2750), §5.7 with Table 8: the
synchronisation-frequency sweep reports, beside the overlap discrepancy of
Eq. (6) and the wall-time ratio, the relative drift of the distance values
outside the overlapping subblocks from the matched independent run.  The pages
give no formula; the reading here:

  * the overlap subblocks of tile k are its upper-left o x o block when it has
    a left neighbour (k > 0) and its lower-right o x o block when it has a
    right neighbour (k < T-1); every other entry of the 64 x 64 map is a
    non-overlap entry;
  * per tile (c, k): num = sum over samples b and non-overlap entries of
    |S - V|, den = the same sum of |V|, with S the synchronised and V the
    independent maps of the same seeds;
  * the relative drift of a chain is sum_k num / sum_k den (a ratio of sums,
    which stays defined on the zero diagonal).
"""
from __future__ import annotations

import numpy as np


def nonoverlap_mask(T: int, k: int, overlap: int = 12, n: int = 64) -> np.ndarray:
    """Boolean ``[n][n]``: True on the non-overlap entries of tile k of T."""
    m = np.ones((n, n), dtype=bool)
    if k > 0:
        m[:overlap, :overlap] = False
    if k < T - 1:
        m[n - overlap:, n - overlap:] = False
    return m


def drift_sums(S: np.ndarray, V: np.ndarray, overlap: int = 12) -> np.ndarray:
    """``S, V [C][T][B][64][64]`` -> ``[C][T][2]`` = (sum |S - V|, sum |V|)
    over the samples and the non-overlap entries of each tile."""
    C, T = S.shape[:2]
    out = np.zeros((C, T, 2))
    for k in range(T):
        m = nonoverlap_mask(T, k, overlap, S.shape[-1])
        Sk = np.asarray(S[:, k], dtype=np.float64)
        Vk = np.asarray(V[:, k], dtype=np.float64)
        out[:, k, 0] = np.abs(Sk - Vk)[..., m].sum(axis=(1, 2))
        out[:, k, 1] = np.abs(Vk)[..., m].sum(axis=(1, 2))
    return out


def relative_drift(S: np.ndarray, V: np.ndarray, overlap: int = 12) -> np.ndarray:
    """Per chain ``[C]``: sum_k num / sum_k den."""
    s = drift_sums(S, V, overlap)
    return s[:, :, 0].sum(axis=1) / s[:, :, 1].sum(axis=1)
