"""GPU noise primitives against the oracle: Philox words bit for bit, and the
float32 Box-Muller transform's error measured over every value of each uniform.

The transform's radius depends only on the first word's top 23 bits and its
angle only on the second word's, so two sweeps of 2^23 values each cover every
input the kernels can see.  The bounds asserted here are the ones the parity
tolerances of the noise fields are derived from:
    |dr|              <= R_ERR            (all radii, r <= sqrt(46 ln 2) = 5.65)
    |d cos|, |d sin|  <= ANG_ERR
    |dz| <= R_ERR + 5.65 ANG_ERR
"""
import numpy as np
import pytest

from oracle import philox
from tests.gpu_util import host, needs_gpu, torch

pytestmark = [pytest.mark.gpu, needs_gpu]

R_ERR = 4e-6
ANG_ERR = 1.5e-6


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


def _u32(a):
    return torch.from_numpy(np.asarray(a, dtype=np.uint32).view(np.int32)).cuda().view(torch.uint32)


def test_philox_words_bit_exact(tdm):
    rng = np.random.default_rng(0)
    n = 1 << 18
    ctr = rng.integers(0, 2**32, size=(n, 4), dtype=np.uint64)
    ctr[:4] = [[0, 0, 0, 0], [0xFFFFFFFF] * 4, [1, 2, 3, 4], [0x80000000, 0, 0x7FFFFFFF, 1]]
    for seed in (0, 1, 0xDEADBEEFCAFEF00D, 2**64 - 1):
        out = torch.empty(n * 4, dtype=torch.uint32, device="cuda")
        tdm.philox4x32(_u32(ctr.astype(np.uint32)).reshape(-1), seed, out)
        got = out.view(torch.int32).cpu().numpy().view(np.uint32).reshape(n, 4).astype(np.uint64)
        ref = np.stack(philox.philox4x32_10(ctr[:, 0], ctr[:, 1], ctr[:, 2], ctr[:, 3],
                                            seed & 0xFFFFFFFF, seed >> 32), axis=1)
        np.testing.assert_array_equal(got, ref)


def _bm(tdm, a, b):
    words = np.stack([a, b], axis=1).astype(np.uint32).reshape(-1)
    z = torch.empty(words.size, device="cuda")
    tdm.box_muller(_u32(words), z)
    return host(z).reshape(-1, 2)


def test_box_muller_radius_all_inputs(tdm):
    m = np.arange(1 << 23, dtype=np.uint64)
    low = np.random.default_rng(1).integers(0, 512, size=m.size, dtype=np.uint64)
    a = (m << np.uint64(9)) | low
    b = np.zeros_like(a)                      # angle 0: z0 = r, z1 = 0
    z = _bm(tdm, a, b)
    r_ref, _ = philox.box_muller(a, b)
    dr = np.abs(z[:, 0] - r_ref)
    print(f"\nmax |dr| = {dr.max():.3e} at r = {r_ref[np.argmax(dr)]:.4g}; "
          f"max |dr|/r (r > 0) = {(dr[1:] / r_ref[1:]).max():.3e}")
    assert dr.max() <= R_ERR
    assert np.abs(z[:, 1]).max() <= ANG_ERR * r_ref.max()


def test_box_muller_angle_all_inputs(tdm):
    k = np.arange(1 << 23, dtype=np.uint64)
    b = (k << np.uint64(9)) | np.uint64(0x1FF)
    a = np.full_like(b, np.uint64(1) << np.uint64(31))   # u1 = 1/2: r = sqrt(2 ln 2)
    z = _bm(tdm, a, b)
    z0, z1 = philox.box_muller(a, b)
    r = np.sqrt(2.0 * np.log(2.0))
    dc, ds = np.abs(z[:, 0] - z0) / r, np.abs(z[:, 1] - z1) / r
    print(f"\nmax |dcos| = {dc.max():.3e}, max |dsin| = {ds.max():.3e}")
    assert dc.max() <= ANG_ERR + R_ERR / r and ds.max() <= ANG_ERR + R_ERR / r
