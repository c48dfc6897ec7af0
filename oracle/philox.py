"""Counter-based normals for the stand-in noise (oracle side, float64).

Philox4x32-10 is written from its published definition: Salmon, Moraes, Dror,
Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC'11 (the Philox-4x32
S-box: two 32x32->64 multiplies per round by 0xD2511F53 and 0xCD9E8D57, the
high halves xored with the other two counter words and the round key, the key
bumped by the Weyl constants 0x9E3779B9 / 0xBB67AE85 between rounds).

The ParaChromo paper says only that samples differ through their noise (§3.3)
and that the per-step noise is keyed by sample and step; the layout below is a
reading of that, written out in the design notes:

  key     = (seed mod 2^32, seed div 2^32)
  counter = (row*16 + quad, step word, g mod 2^32, (g div 2^32 mod 2^24) | tag<<24)

where ``g`` is the map's global sample id, ``tag`` the noise stream and
``(row, quad)`` a row-aligned group of four columns ``4*quad .. 4*quad+3``.
Each output word pair (a, b) gives two normals by Box-Muller on 23-bit
uniforms u1 = 1 - (a>>9) / 2^23 in (0, 1] and u2 = (b>>9) / 2^23 in [0, 1):
r = sqrt(-2 ln u1), z0 = r cos(2 pi u2), z1 = r sin(2 pi u2).  (23 bits: both
uniforms are then exact float32 numbers built from a float's mantissa.)
"""
from __future__ import annotations

import numpy as np

MASK32 = np.uint64(0xFFFFFFFF)
PHILOX_M0 = np.uint64(0xD2511F53)
PHILOX_M1 = np.uint64(0xCD9E8D57)
PHILOX_W0 = np.uint64(0x9E3779B9)
PHILOX_W1 = np.uint64(0xBB67AE85)

# noise streams
TAG_INIT = 0    # initial state x_T
TAG_EPS_C = 1   # conditional eps stream of the stand-in
TAG_EPS_U = 2   # unconditional eps stream of the stand-in
TAG_ETA = 3     # the sigma_i z term of DDIM with eta > 0

N = 64
N_QUADS = N // 4


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Ten Philox-4x32 rounds on broadcastable arrays of 32-bit values.

    Inputs are any integer arrays (values < 2^32); the four output words come
    back as uint64 arrays holding 32-bit values.
    """
    c0, c1, c2, c3, k0, k1 = (np.asarray(v, dtype=np.uint64) & MASK32
                              for v in (c0, c1, c2, c3, k0, k1))
    c0, c1, c2, c3, k0, k1 = np.broadcast_arrays(c0, c1, c2, c3, k0, k1)
    for _ in range(10):
        p0 = PHILOX_M0 * c0          # < 2^64: exact in uint64
        p1 = PHILOX_M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
        k0 = (k0 + PHILOX_W0) & MASK32
        k1 = (k1 + PHILOX_W1) & MASK32
    return c0, c1, c2, c3


def box_muller(a, b):
    """Two standard normals from two 32-bit words (float64)."""
    a = np.asarray(a, dtype=np.uint64)
    b = np.asarray(b, dtype=np.uint64)
    u1 = 1.0 - (a >> np.uint64(9)).astype(np.float64) / 8388608.0
    u2 = (b >> np.uint64(9)).astype(np.float64) / 8388608.0
    r = np.sqrt(-2.0 * np.log(u1))
    return r * np.cos(2.0 * np.pi * u2), r * np.sin(2.0 * np.pi * u2)


def upper_quads():
    """(row, quad) of every row-aligned column quad touching the upper triangle.

    Row r, quad q covers columns 4q..4q+3 and is kept when 4q+3 >= r: 544 quads
    for 64 beads.  Entries (r, j) with j < r inside a kept quad are drawn but
    never used.
    """
    rows, quads = [], []
    for r in range(N):
        for q in range(N_QUADS):
            if 4 * q + 3 >= r:
                rows.append(r)
                quads.append(q)
    return np.array(rows, dtype=np.int64), np.array(quads, dtype=np.int64)


def counters(g, tag: int, step_word: int, rows, quads):
    """Philox counter words for maps with sample ids ``g`` (shape [M]) at the
    given (row, quad) positions (shape [Q]); result broadcasts to [M, Q]."""
    g = np.asarray(g, dtype=np.uint64).reshape(-1, 1)
    c0 = (rows.astype(np.uint64) << np.uint64(4)) | quads.astype(np.uint64)
    c0 = c0.reshape(1, -1)
    c1 = np.uint64(step_word & 0xFFFFFFFF)
    c2 = g & MASK32
    c3 = ((g >> np.uint64(32)) & np.uint64(0xFFFFFF)) | np.uint64((tag & 0xFF) << 24)
    return c0, c1, c2, c3


def symmetric_normal(seed: int, tag: int, step_word: int, g) -> np.ndarray:
    """The symmetric N(0,1) field ``[M, 64, 64]`` of one stream and step.

    Entry (i, j) with i <= j is the Box-Muller normal of its own row quad;
    entry (i, j) with i > j equals entry (j, i).  The diagonal is an ordinary
    entry.  This keeps a state that starts symmetric symmetric, matching the
    folded state that holds each bead pair once (ParaChromo §3.1, §4.3.2).
    """
    rows, quads = upper_quads()
    c0, c1, c2, c3 = counters(g, tag, step_word, rows, quads)
    k0 = np.uint64(seed & 0xFFFFFFFF)
    k1 = np.uint64((seed >> 32) & 0xFFFFFFFF)
    w0, w1, w2, w3 = philox4x32_10(c0, c1, c2, c3, k0, k1)
    za, zb = box_muller(w0, w1)
    zc, zd = box_muller(w2, w3)
    m = c2.shape[0]
    z = np.zeros((m, N, N), dtype=np.float64)
    cols = 4 * quads
    z[:, rows, cols] = za
    z[:, rows, cols + 1] = zb
    z[:, rows, cols + 2] = zc
    z[:, rows, cols + 3] = zd
    upper = np.triu(z)
    return upper + np.swapaxes(np.triu(z, 1), -1, -2)
