"""Helpers for the GPU parity tests (tolerances, device transfers, inputs)."""
import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

# Tolerances (normwise per map: max |gpu - oracle| / max |oracle|)
TOL_MAP = 1e-5        # final and intermediate sampler states
# absolute bound on one float32 normal against float64: |dr| + r_max |d angle|
# with the exhaustively measured bounds of tests/test_gpu_noise.py
Z_ABS_ERR = 4e-6 + 5.65 * 1.5e-6
TOL_RECOVER = 1e-4    # distance maps rebuilt from MDS coordinates; eigenvalues
TOL_SEAM = 1e-4       # seam discrepancy, relative with a floor


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host(t):
    return t.detach().cpu().numpy().astype(np.float64)


def normwise(g, o):
    """Per-map normwise relative error over the last two axes."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    num = np.abs(g - o).max(axis=(-1, -2))
    den = np.maximum(np.abs(o).max(axis=(-1, -2)), 1e-30)
    return num / den


def assert_maps_close(g, o, tol=TOL_MAP, what="maps"):
    e = normwise(g, o)
    worst = np.unravel_index(np.argmax(e), e.shape)
    assert e.max() <= tol, f"{what}: normwise error {e.max():.3e} > {tol:.1e} at {worst}"
    return e.max()


def x0_disagreeing(seed, C, T):
    """Chain reference maps plus a symmetric per-tile perturbation, so that the
    overlap blocks of adjacent tiles differ and the projection's x0 term is
    exercised (the chain maps alone agree on every overlap)."""
    x0 = synth.chain_x0(seed, C, T).astype(np.float64)
    p = np.random.default_rng([seed, 404]).uniform(-0.5, 0.5, size=x0.shape)
    return (x0 + 0.5 * (p + np.swapaxes(p, -1, -2))).astype(np.float32)
