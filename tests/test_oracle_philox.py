"""Pins of the oracle's counter-based noise against things other than itself."""
import json
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest

from oracle import philox

TRITON_SCRIPT = textwrap.dedent(r"""
    import os, sys, json
    os.environ["TRITON_INTERPRET"] = "1"
    import torch, triton, triton.language as tl

    @triton.jit
    def kern(out_ptr, c_ptr, k_ptr, n: tl.constexpr):
        i = tl.arange(0, n)
        c0 = tl.load(c_ptr + 0 * n + i)
        c1 = tl.load(c_ptr + 1 * n + i)
        c2 = tl.load(c_ptr + 2 * n + i)
        c3 = tl.load(c_ptr + 3 * n + i)
        k0 = tl.load(k_ptr + 0 * n + i)
        k1 = tl.load(k_ptr + 1 * n + i)
        a, b, c, d = tl.philox_impl(c0, c1, c2, c3, k0, k1, 10)
        tl.store(out_ptr + 0 * n + i, a)
        tl.store(out_ptr + 1 * n + i, b)
        tl.store(out_ptr + 2 * n + i, c)
        tl.store(out_ptr + 3 * n + i, d)

    data = json.loads(sys.stdin.read())
    n = len(data["c"][0])
    c = torch.tensor(data["c"], dtype=torch.int64).to(torch.uint32).flatten()
    k = torch.tensor(data["k"], dtype=torch.int64).to(torch.uint32).flatten()
    out = torch.zeros(4 * n, dtype=torch.uint32)
    kern[(1,)](out, c, k, n)
    print(json.dumps(out.to(torch.int64).view(4, n).tolist()))
""")


def _triton_philox(c, k):
    """Philox4x32-10 from triton's library implementation, run by its CPU
    interpreter in a child process (so the interpreter flag stays local)."""
    env = dict(os.environ, TRITON_INTERPRET="1")
    res = subprocess.run([sys.executable, "-c", TRITON_SCRIPT], input=json.dumps({"c": c, "k": k}),
                         capture_output=True, text=True, env=env, timeout=600)
    if res.returncode != 0:
        pytest.skip(f"triton interpreter unavailable: {res.stderr[-400:]}")
    return np.array(json.loads(res.stdout.strip().splitlines()[-1]), dtype=np.uint64)


def test_philox_matches_triton_library():
    rng = np.random.default_rng(1234)
    n = 64
    c = rng.integers(0, 2**32, size=(4, n), dtype=np.uint64)
    k = rng.integers(0, 2**32, size=(2, n), dtype=np.uint64)
    # edge words
    c[:, 0] = 0
    k[:, 0] = 0
    c[:, 1] = 0xFFFFFFFF
    k[:, 1] = 0xFFFFFFFF
    c[:, 2] = [0, 1, 2, 3]
    ref = _triton_philox(c.astype(np.int64).tolist(), k.astype(np.int64).tolist())
    got = np.stack(philox.philox4x32_10(c[0], c[1], c[2], c[3], k[0], k[1]))
    np.testing.assert_array_equal(got, ref)


def test_box_muller_special_values():
    # a>>9 = 0 -> u1 = 1 -> r = 0
    z0, z1 = philox.box_muller(0x000001FF, 12345 << 9)
    assert z0 == 0.0 and z1 == 0.0
    # a>>9 = 2^23 - 1 -> u1 = 2^-23 -> r = sqrt(2 * 23 ln 2); b = 0 -> angle 0
    r = np.sqrt(46.0 * np.log(2.0))
    z0, z1 = philox.box_muller(0xFFFFFFFF, 0)
    assert abs(z0 - r) < 1e-14 and z1 == 0.0
    # b>>9 = 2^21 -> u2 = 1/4 -> angle pi/2
    z0, z1 = philox.box_muller(0xFFFFFFFF, 1 << 30)
    assert abs(z0) < 1e-14 and abs(z1 - r) < 1e-14
    # b>>9 = 2^22 -> u2 = 1/2 -> angle pi
    z0, z1 = philox.box_muller(0xFFFFFFFF, 1 << 31)
    assert abs(z0 + r) < 1e-14 and abs(z1) < 1e-14
    # a>>9 = 2^22 -> u1 = 1/2 -> r = sqrt(2 ln 2)
    z0, _ = philox.box_muller(1 << 31, 0)
    assert abs(z0 - np.sqrt(2.0 * np.log(2.0))) < 1e-15
    # the low 9 bits of either word are ignored
    assert philox.box_muller(0x12345678, 0x9ABCDEF0) == philox.box_muller(0x123457FF, 0x9ABCDE00)


def test_normals_are_standard():
    from scipy import stats
    g = np.arange(500, dtype=np.uint64)
    z = philox.symmetric_normal(7, philox.TAG_EPS_C, 3, g)
    iu = np.triu_indices(64)
    v = z[:, iu[0], iu[1]].ravel()          # the independent entries
    assert v.size == 500 * 2080
    assert abs(v.mean()) < 5.0 / np.sqrt(v.size)
    assert abs(v.var() - 1.0) < 6.0 * np.sqrt(2.0 / v.size)
    assert stats.kstest(v[:200000], "norm").pvalue > 1e-4
    # the tail is cut at r = sqrt(46 ln 2) ~ 5.65
    assert np.abs(v).max() <= np.sqrt(46.0 * np.log(2.0)) + 1e-12


def test_streams_steps_and_samples_are_independent():
    g = np.arange(200, dtype=np.uint64)
    iu = np.triu_indices(64)
    fields = [philox.symmetric_normal(11, philox.TAG_EPS_C, 5, g),
              philox.symmetric_normal(11, philox.TAG_EPS_U, 5, g),
              philox.symmetric_normal(11, philox.TAG_EPS_C, 6, g),
              philox.symmetric_normal(11, philox.TAG_EPS_C, 5, g + np.uint64(1 << 40)),
              philox.symmetric_normal(12, philox.TAG_EPS_C, 5, g)]
    flat = [f[:, iu[0], iu[1]].ravel() for f in fields]
    for i in range(len(flat)):
        for j in range(i + 1, len(flat)):
            r = np.corrcoef(flat[i], flat[j])[0, 1]
            assert abs(r) < 5.0 / np.sqrt(flat[i].size), (i, j, r)
    # neighbouring samples inside one field are uncorrelated too
    r = np.corrcoef(flat[0].reshape(200, -1)[:-1].ravel(), flat[0].reshape(200, -1)[1:].ravel())[0, 1]
    assert abs(r) < 5.0 / np.sqrt(flat[0].size)


def test_symmetric_field_structure():
    g = np.array([0, 1, 2**35 + 17], dtype=np.uint64)
    z = philox.symmetric_normal(3, philox.TAG_INIT, 0, g)
    assert z.shape == (3, 64, 64)
    np.testing.assert_array_equal(z, np.swapaxes(z, -1, -2))
    assert np.all(np.diagonal(z, axis1=1, axis2=2) != 0.0)
    # deterministic
    np.testing.assert_array_equal(z, philox.symmetric_normal(3, philox.TAG_INIT, 0, g))
    # 544 row quads cover the upper triangle
    rows, quads = philox.upper_quads()
    assert len(rows) == 544
    covered = np.zeros((64, 64), dtype=bool)
    for r, q in zip(rows, quads):
        covered[r, 4 * q:4 * q + 4] = True
    assert np.all(covered[np.triu_indices(64)])
