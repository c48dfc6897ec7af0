"""GPU parity of the sampler path (init noise, stand-in eps, DDIM step, fused
run) against the float64 oracle, through the C ABI."""
import numpy as np
import pytest

import synth
from oracle import philox, schedule as osched
from oracle.ddim import (ddim_run as o_run, eps_standin as o_eps, init_noise as o_init,
                         sample_ids, stream_noise)
from tests.gpu_util import (TOL_MAP, Z_ABS_ERR, assert_maps_close, dev, host, needs_gpu, normwise, torch,
                            x0_disagreeing)

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(scope="module")
def tdm():
    import tiled_distance_maps_b200 as m
    return m


def _maps(tiling):
    return torch.empty(tiling.n_maps * 4096, device="cuda", dtype=torch.float32)


def _as5(t, tiling):
    return host(t).reshape(tiling.C, tiling.T, tiling.B, 64, 64)


def test_schedule_table_matches_oracle(tdm):
    for S, eta in ((50, 0.0), (1000, 1.0), (250, 0.5)):
        if 1000 % S:
            continue
        tab = np.array(tdm.Schedule(S, eta).table())
        o = osched.Schedule(S=S, eta=eta)
        np.testing.assert_array_equal(tab[:, 0], o.tau)
        np.testing.assert_allclose(tab[:, 1], o.ab_t, rtol=1e-14)
        np.testing.assert_allclose(tab[:, 2], o.ab_p, rtol=1e-14)
        np.testing.assert_allclose(tab[:, 3], o.sigma, rtol=1e-12, atol=1e-15)


def test_cosine_schedule(tdm):
    # the library's cosine table (Nichol & Dhariwal) against the oracle's, the
    # DDIM table built from it, and a fused run on it
    for T_train, s in ((1000, 0.008), (1200, 0.0), (7, 0.1)):
        np.testing.assert_allclose(tdm.cosine_alphas_bar(T_train, s), osched.cosine_alphas_bar(T_train, s),
                                   rtol=1e-13)
    ab = tdm.cosine_alphas_bar(1000)
    oab = osched.cosine_alphas_bar(1000)
    for S, eta in ((50, 0.0), (250, 1.0)):
        tab = np.array(tdm.Schedule(S, eta, alphas_bar=ab).table())
        o = osched.Schedule(S=S, eta=eta, alphas_bar_table=oab)
        np.testing.assert_array_equal(tab[:, 0], o.tau)
        np.testing.assert_allclose(tab[:, 1], o.ab_t, rtol=1e-13)
        np.testing.assert_allclose(tab[:, 2], o.ab_p, rtol=1e-13)
        np.testing.assert_allclose(tab[:, 3], o.sigma, rtol=1e-11, atol=1e-15)
    t = tdm.Tiling(C=1, T=4, B=8, overlap=12, sync_every=1)
    x0 = synth.chain_x0(0, 1, 4)
    maps = _maps(t)
    tdm.ddim_run(tdm.Schedule(50, eta=1.0, alphas_bar=ab), maps, dev(x0), 1.0, 0.1, 0.3, 0, t)
    ref = o_run(x0, osched.Schedule(S=50, eta=1.0, alphas_bar_table=oab), 1.0, 0.1, 0.3, 0, np.arange(8), 8)
    assert_maps_close(_as5(maps, t), ref, TOL_MAP, "fused run on the cosine schedule")
    with pytest.raises(tdm.TdmError):
        tdm.cosine_alphas_bar(0)


@pytest.mark.parametrize("base,boff", [(0, 0), (12345, 3)])
def test_init_noise(tdm, base, boff):
    t = tdm.Tiling(C=2, T=3, B=4, B_total=9, b_offset=boff, sample_id_base=base)
    m = _maps(t)
    tdm.init_noise(m, t, seed=0xDEADBEEF12345)
    g = _as5(m, t)
    ids = sample_ids(2, 3, np.arange(boff, boff + 4), 9, base)
    ref = o_init(0xDEADBEEF12345, ids)
    assert np.abs(g - ref).max() <= Z_ABS_ERR
    np.testing.assert_array_equal(g, np.swapaxes(g, -1, -2))


@pytest.mark.parametrize("tag,s", [(1, 0.1), (2, 0.3)])
def test_eps_standin(tdm, tag, s):
    t = tdm.Tiling(C=1, T=2, B=3)
    sch = tdm.Schedule(50)
    o = osched.Schedule(S=50)
    x = synth.gaussian_maps(4, 6, symmetric=False).reshape(1, 2, 3, 64, 64) * 3.0
    x0 = synth.chain_x0(1, 1, 2)
    out = _maps(t)
    for step in (49, 20, 0):
        tdm.eps_standin(sch, step, dev(x), dev(x0), s, tag, 77, t, out)
        z = stream_noise(77, tag, step, sample_ids(1, 2, np.arange(3), 3))
        ref = o_eps(x.astype(np.float64), x0[:, :, None].astype(np.float64), o.ab_t[step], s, z)
        assert_maps_close(_as5(out, t), ref, 1e-5, f"eps step {step}")


def _gpu_per_step(tdm, sch, x0, t, w, s_c, s_u, seed, xT=None):
    """The step-by-step path: init noise, then per step the stand-in eps of
    each stream and one DDIM step (with the projection when it is due)."""
    maps = _maps(t)
    if xT is None:
        tdm.init_noise(maps, t, seed)
    else:
        maps.copy_(dev(xT).reshape(-1))
    ec, eu = _maps(t), (_maps(t) if w != 0 else None)
    x0d = dev(x0)
    states = []
    for i in reversed(range(sch.S)):
        tdm.eps_standin(sch, i, maps, x0d, s_c, tdm.STREAM_EPS_C, seed, t, ec)
        if w != 0:
            tdm.eps_standin(sch, i, maps, x0d, s_u, tdm.STREAM_EPS_U, seed, t, eu)
        tdm.ddim_step(sch, i, maps, ec, eu, w, seed, t)
        states.append(_as5(maps, t))
    return states


def test_per_step_path_small_chain(tdm):
    # 1 chain x 4 tiles x 8 samples, 50 steps, eta 0, w 0, eps_c noise 0.1,
    # projection after every step
    wl = synth.WORKLOADS["chain4_b8_s50"]
    t = tdm.Tiling(C=1, T=4, B=8, overlap=12, sync_every=1)
    sch = tdm.Schedule(50)
    x0 = synth.chain_x0(wl.seed, 1, 4)
    got = _gpu_per_step(tdm, sch, x0, t, 0.0, 0.1, 0.3, wl.seed)
    _, traj = o_run(x0, osched.Schedule(S=50), 0.0, 0.1, 0.3, wl.seed, np.arange(8), 8, return_trajectory=True)
    for n, (g, o) in enumerate(zip(got, traj)):
        assert_maps_close(g, o, TOL_MAP, f"state after step {n + 1}")


def test_per_step_path_cfg_eta_unsymmetric_start(tdm):
    # w = 1 and eta = 1 exercise both eps streams and the eta stream; a start
    # that is not symmetric checks that every entry is updated on its own
    t = tdm.Tiling(C=2, T=3, B=2, overlap=8, sync_every=2)
    sch = tdm.Schedule(10, eta=1.0)
    x0 = synth.chain_x0(3, 2, 3, overlap=8)
    xT = synth.gaussian_maps(9, 12, symmetric=False).reshape(2, 3, 2, 64, 64)
    got = _gpu_per_step(tdm, sch, x0, t, 1.0, 0.1, 0.3, 5, xT=xT)
    _, traj = _oracle_unfolded(x0, 10, 1.0, 1.0, 0.1, 0.3, 5, 2, 8, 2, xT)
    for n, (g, o) in enumerate(zip(got, traj)):
        assert_maps_close(g, o, TOL_MAP, f"state after step {n + 1}")


def _oracle_unfolded(x0, S, eta, w, s_c, s_u, seed, B, overlap, K, xT):
    """The oracle run on a full (not folded) start state: same steps as
    oracle.ddim.ddim_run without the fold of x_T."""
    from oracle.ddim import cfg_combine, ddim_update
    from oracle.seam import seam_project
    o = osched.Schedule(S=S, eta=eta)
    C, T = x0.shape[:2]
    g = sample_ids(C, T, np.arange(B), B)
    x = xT.astype(np.float64)
    x0b = x0[:, :, None].astype(np.float64)
    traj = []
    for i in reversed(range(S)):
        e = o_eps(x, x0b, o.ab_t[i], s_c, stream_noise(seed, philox.TAG_EPS_C, i, g))
        if w != 0:
            e = cfg_combine(e, o_eps(x, x0b, o.ab_t[i], s_u, stream_noise(seed, philox.TAG_EPS_U, i, g)), w)
        z = stream_noise(seed, philox.TAG_ETA, i, g) if eta > 0 else None
        x = ddim_update(x, e, o.ab_t[i], o.ab_p[i], o.sigma[i], z)
        if T > 1 and K > 0 and (S - i) % K == 0:
            x = seam_project(x, overlap)
        traj.append(x.copy())
    return x, traj


def test_fused_run_small_chain(tdm):
    wl = synth.WORKLOADS["chain4_b8_s50"]
    t = tdm.Tiling(C=1, T=4, B=8, overlap=12, sync_every=1)
    sch = tdm.Schedule(50)
    x0 = synth.chain_x0(wl.seed, 1, 4)
    maps = _maps(t)
    tdm.ddim_run(sch, maps, dev(x0), 0.0, 0.1, 0.3, wl.seed, t)
    ref = o_run(x0, osched.Schedule(S=50), 0.0, 0.1, 0.3, wl.seed, np.arange(8), 8)
    g = _as5(maps, t)
    assert_maps_close(g, ref, TOL_MAP, "fused final maps")
    np.testing.assert_array_equal(g, np.swapaxes(g, -1, -2))
    # the final overlap blocks agree exactly after the last projection
    np.testing.assert_array_equal(g[:, :-1, :, 52:, 52:], g[:, 1:, :, :12, :12])


@pytest.mark.parametrize("overlap,K,S,eta,w,T", [(12, 1, 10, 1.0, 0.5, 3), (4, 3, 20, 0.0, 1.0, 4),
                                                 (32, 2, 5, 1.0, 0.0, 2), (12, 0, 8, 0.0, 1.0, 3),
                                                 (12, 1, 4, 0.0, 1.0, 1)])
def test_fused_run_variants_given_start(tdm, overlap, K, S, eta, w, T):
    C, B = 2, 5
    t = tdm.Tiling(C=C, T=T, B=B, overlap=overlap, sync_every=K)
    sch = tdm.Schedule(S, eta=eta)
    x0 = synth.chain_x0(11, C, T, overlap=overlap)
    xT = synth.gaussian_maps(13, C * T * B, symmetric=False).reshape(C, T, B, 64, 64)
    maps = dev(xT).reshape(-1).clone()
    tdm.ddim_run(sch, maps, dev(x0), w, 0.1, 0.3, 21, t, init_noise=False)
    ref = o_run(x0, osched.Schedule(S=S, eta=eta), w, 0.1, 0.3, 21, np.arange(B), B, overlap=overlap,
                sync_every=K, x_T=xT)
    assert_maps_close(_as5(maps, t), ref, TOL_MAP, "fused final maps")


def test_fused_equals_per_step_on_symmetric_start(tdm):
    t = tdm.Tiling(C=1, T=3, B=4, overlap=12, sync_every=1)
    sch = tdm.Schedule(25, eta=1.0)
    x0 = synth.chain_x0(2, 1, 3)
    fused = _maps(t)
    tdm.ddim_run(sch, fused, dev(x0), 1.0, 0.1, 0.3, 8, t)
    states = _gpu_per_step(tdm, sch, x0, t, 1.0, 0.1, 0.3, 8)
    assert normwise(_as5(fused, t), states[-1]).max() < 2 * TOL_MAP
    # and a state before the last step (which alone sets the final maps)
    for m in (5, 24):
        part = _maps(t)
        tdm.ddim_run(sch, part, dev(x0), 1.0, 0.1, 0.3, 8, t, first_step=24, n_steps=m)
        assert normwise(_as5(part, t), states[m - 1]).max() < 2 * TOL_MAP, m


def test_fused_run_is_deterministic_and_shards_reproduce_it(tdm):
    t = tdm.Tiling(C=1, T=4, B=6, overlap=12, sync_every=1)
    sch = tdm.Schedule(20)
    x0 = dev(synth.chain_x0(5, 1, 4))
    a, b = _maps(t), _maps(t)
    tdm.ddim_run(sch, a, x0, 1.0, 0.1, 0.3, 3, t)
    tdm.ddim_run(sch, b, x0, 1.0, 0.1, 0.3, 3, t)
    torch.testing.assert_close(a, b, rtol=0, atol=0)
    full = a.view(1, 4, 6, 4096)
    for b0, nb in ((0, 2), (2, 3), (5, 1)):
        ts = tdm.Tiling(C=1, T=4, B=nb, overlap=12, sync_every=1, B_total=6, b_offset=b0)
        part = torch.empty(4 * nb * 4096, device="cuda")
        tdm.ddim_run(sch, part, x0, 1.0, 0.1, 0.3, 3, ts)
        torch.testing.assert_close(part.view(1, 4, nb, 4096), full[:, :, b0:b0 + nb], rtol=0, atol=0)


def test_chromosome_chain_full_size_sampled(tdm):
    # 32 tiles x 1000 samples, CFG w=1 (eps_c noise 0.1, eps_u noise 0.3),
    # 50 steps, projection every step: the launch the benchmark times
    wl = synth.WORKLOADS["chain32_b1000_cfg"]
    t = tdm.Tiling(C=1, T=32, B=1000, overlap=12, sync_every=1)
    sch = tdm.Schedule(50)
    x0 = synth.chain_x0(wl.seed, 1, 32, sigma=wl.sigma)
    maps = _maps(t)
    tdm.ddim_run(sch, maps, dev(x0), wl.w, wl.s_c, wl.s_u, wl.seed, t)
    g = maps.view(1, 32, 1000, 64, 64)
    refs = {}
    for b in (0, 417, 999):
        refs[b] = o_run(x0, osched.Schedule(S=50), wl.w, wl.s_c, wl.s_u, wl.seed, [b], 1000, return_trajectory=True)
        assert_maps_close(host(g[:, :, b:b + 1]), refs[b][0], TOL_MAP, f"sample {b}")
    assert torch.isfinite(g).all()
    # the same launch stopped before the last step, which alone sets the final maps
    tdm.ddim_run(sch, maps, dev(x0), wl.w, wl.s_c, wl.s_u, wl.seed, t, first_step=49, n_steps=49)
    for b in (0, 417, 999):
        assert_maps_close(host(g[:, :, b:b + 1]), refs[b][1][48], TOL_MAP, f"sample {b}, 49 steps")


def test_invalid_arguments_are_rejected(tdm):
    t = tdm.Tiling(C=1, T=2, B=1, overlap=12)
    sch = tdm.Schedule(10)
    m = _maps(t)
    x0 = torch.zeros(2 * 4096, device="cuda")
    with pytest.raises(tdm.TdmError) as e:
        tdm.ddim_run(sch, m, x0, 0.0, 0.1, 0.3, 0, tdm.Tiling(C=1, T=2, B=1, overlap=10))
    assert e.value.status == tdm.EUNSUPPORTED
    with pytest.raises(tdm.TdmError) as e:
        tdm.ddim_run(sch, m, x0, 0.0, 0.1, 0.3, 0, tdm.Tiling(C=1, T=2, B=1, overlap=40))
    assert e.value.status == tdm.EINVAL
    with pytest.raises(tdm.TdmError) as e:
        tdm.ddim_step(sch, 10, m, m, None, 0.0, 0, t)
    assert e.value.status == tdm.EINVAL
    with pytest.raises(tdm.TdmError) as e:
        tdm.ddim_step(sch, 3, m, m, None, 1.0, 0, t)
    assert e.value.status == tdm.EINVAL
    with pytest.raises(tdm.TdmError) as e:
        tdm.Schedule(30)
    assert e.value.status == tdm.EINVAL
    with pytest.raises(tdm.TdmError) as e:
        tdm.ddim_run(sch, m[1:], x0, 0.0, 0.1, 0.3, 0, tdm.Tiling(C=1, T=1, B=1))
    assert e.value.status == tdm.EINVAL       # misaligned pointer
    # empty batches are a no-op
    tdm.ddim_run(sch, m, x0, 0.0, 0.1, 0.3, 0, tdm.Tiling(C=0, T=2, B=1))
    tdm.ddim_run(sch, m, x0, 0.0, 0.1, 0.3, 0, tdm.Tiling(C=1, T=2, B=0))


def test_ddpm_ancestral_sampler_1000_steps(tdm):
    # DDIM at eta = 1 with every training timestep is the DDPM ancestral
    # sampler (posterior variance beta-tilde) used by the synchronisation
    # experiments: the fused run against an oracle loop of DDPM steps
    from oracle.ddim import ddpm_ancestral_step, eps_standin as oe, init_noise as oi
    from oracle.seam import seam_project
    T, B, S = 3, 2, 1000
    t = tdm.Tiling(C=1, T=T, B=B, overlap=12, sync_every=1)
    sch = tdm.Schedule(S, eta=1.0)
    x0 = synth.chain_x0(17, 1, T)
    maps = _maps(t)
    tdm.ddim_run(sch, maps, dev(x0), 1.0, 0.1, 0.3, 23, t)
    o = osched.Schedule(S=S, eta=1.0)
    g = sample_ids(1, T, np.arange(B), B)
    x = oi(23, g)
    x0b = x0[:, :, None].astype(np.float64)
    for tt in reversed(range(S)):
        ec = oe(x, x0b, o.ab[tt], 0.1, stream_noise(23, philox.TAG_EPS_C, tt, g))
        eu = oe(x, x0b, o.ab[tt], 0.3, stream_noise(23, philox.TAG_EPS_U, tt, g))
        x = ddpm_ancestral_step(x, 2.0 * ec - eu, tt, o.betas, o.ab, stream_noise(23, philox.TAG_ETA, tt, g))
        x = seam_project(x)
    assert_maps_close(_as5(maps, t), x, TOL_MAP, "DDPM run")


@pytest.mark.parametrize("S,K,eta,w", [(10, 1, 0.0, 1.0), (10, 3, 1.0, 0.0), (20, 2, 1.0, 1.0), (8, 0, 0.0, 1.0)])
def test_fused_run_intermediate_states(tdm, S, K, eta, w):
    # The stand-in's last step (alpha_bar_prev = 1) gives x0 plus that step's
    # own noise whatever the state before it, so final maps alone do not see
    # the trajectory: the states after m < S steps are compared here, from a
    # single run of m steps and from runs resumed in parts.
    C, T, B = 2, 3, 4
    t = tdm.Tiling(C=C, T=T, B=B, overlap=12, sync_every=K)
    sch = tdm.Schedule(S, eta=eta)
    x0 = x0_disagreeing(11, C, T)
    x0d = dev(x0).reshape(-1)
    _, traj = o_run(x0, osched.Schedule(S=S, eta=eta), w, 0.1, 0.3, 9, np.arange(B), B, overlap=12, sync_every=K,
                    return_trajectory=True)
    for m in (1, 2, S // 2, S - 1, S):
        maps = _maps(t)
        tdm.ddim_run(sch, maps, x0d, w, 0.1, 0.3, 9, t, first_step=S - 1, n_steps=m)
        assert_maps_close(_as5(maps, t), traj[m - 1], TOL_MAP, f"state after {m} of {S} steps")
    for cuts in ((1,), (S // 3, S // 2)):
        parts, done = _maps(t), 0
        for n in list(cuts) + [S - 1]:
            tdm.ddim_run(sch, parts, x0d, w, 0.1, 0.3, 9, t, init_noise=done == 0, first_step=S - 1 - done,
                         n_steps=n - done)
            done = n
        assert_maps_close(_as5(parts, t), traj[S - 2], TOL_MAP, f"state after {S - 1} steps, cut at {cuts}")


@pytest.mark.parametrize("S,K,eta,w,cuts", [(10, 1, 0.0, 1.0, (4,)), (10, 3, 1.0, 0.0, (2, 7)),
                                            (8, 0, 0.0, 1.0, (5,)), (20, 3, 1.0, 1.0, (1, 10, 19))])
def test_fused_run_resumes_bit_exactly(tdm, S, K, eta, w, cuts):
    # the run split after the given numbers of steps, the state kept in the
    # maps between the parts, ends on the whole run's final maps bit for bit
    # (the last step sets them from x0, its own noise and, where projected,
    # the partner's; test_fused_run_intermediate_states covers the states
    # before it)
    t = tdm.Tiling(C=2, T=3, B=4, overlap=12, sync_every=K)
    sch = tdm.Schedule(S, eta=eta)
    x0 = dev(synth.chain_x0(2, 2, 3)).reshape(-1)
    whole = _maps(t)
    tdm.ddim_run(sch, whole, x0, w, 0.1, 0.3, 9, t)
    parts = _maps(t)
    done = 0
    for n in list(cuts) + [S]:
        tdm.ddim_run(sch, parts, x0, w, 0.1, 0.3, 9, t, init_noise=done == 0, first_step=S - 1 - done,
                     n_steps=n - done)
        done = n
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(parts), host(whole))


def test_fused_run_step_range_is_checked(tdm):
    t = tdm.Tiling(C=1, T=2, B=1)
    sch = tdm.Schedule(10)
    x0, m = dev(synth.chain_x0(0, 1, 2)).reshape(-1), _maps(t)
    for first, n, init in ((10, 1, False), (-1, 1, False), (5, 7, False), (5, 0, False), (5, 2, True)):
        with pytest.raises(tdm.TdmError):
            tdm.ddim_run(sch, m, x0, 0.0, 0.1, 0.0, 0, t, init_noise=init, first_step=first, n_steps=n)


def test_large_and_small_launch_shapes_agree(tdm):
    # A launch of at least 4 x 8 warps per SM runs 8-warp CTAs with the
    # warp-voted series; a smaller one runs 2-warp CTAs with the series
    # selected per pair.  Both give the same bits, and the large one matches
    # the oracle (final maps and a state before the last step).
    import torch as _t
    sms = _t.cuda.get_device_properties(0).multi_processor_count
    T, S = 4, 10
    B = -(-4 * 8 * sms // (17 * T))          # enough chain-samples for 8-warp CTAs
    t_big = tdm.Tiling(C=1, T=T, B=B, overlap=12, sync_every=1)
    sch = tdm.Schedule(S)
    x0 = x0_disagreeing(21, 1, T)
    x0d = dev(x0).reshape(-1)
    big = _maps(t_big)
    tdm.ddim_run(sch, big, x0d, 1.0, 0.1, 0.3, 4, t_big)
    part = _maps(t_big)
    tdm.ddim_run(sch, part, x0d, 1.0, 0.1, 0.3, 4, t_big, first_step=S - 1, n_steps=S - 1)
    for off in (0, B - 3):
        t_small = tdm.Tiling(C=1, T=T, B=3, overlap=12, sync_every=1, B_total=B, b_offset=off)
        small = _maps(t_small)
        tdm.ddim_run(sch, small, x0d, 1.0, 0.1, 0.3, 4, t_small)
        np.testing.assert_array_equal(_as5(small, t_small), _as5(big, t_big)[:, :, off:off + 3])
    ref, traj = o_run(x0, osched.Schedule(S=S), 1.0, 0.1, 0.3, 4, np.arange(B), B, overlap=12, sync_every=1,
                      return_trajectory=True)
    assert_maps_close(_as5(big, t_big), ref, TOL_MAP, "large launch, final maps")
    assert_maps_close(_as5(part, t_big), traj[S - 2], TOL_MAP, "large launch, state before the last step")


def test_compute_entry_points_take_no_device_memory_for_new_shapes(tdm):
    # The library allocates only when a context or a schedule is created: the
    # fused run derives its lane map in the kernel, so a new (T, overlap)
    # shape, a per-step call with the projection and a long stitched chain
    # leave the free device memory where it was.  Each kernel variant runs
    # once first (CUDA may load its code lazily on the first launch), and
    # every buffer is allocated before the first reading.
    ctx = tdm.context(0)
    sch = tdm.Schedule(5, ctx=ctx)
    shapes = ((4, 12), (40, 12), (7, 8), (33, 32), (2, 4))
    x0s = {(T, o): dev(synth.chain_x0(2, 1, T, overlap=o)).reshape(-1) for T, o in shapes}
    maps = torch.empty(40 * 3 * 4096, device="cuda")
    eps = torch.zeros_like(maps)
    coords = torch.empty(40 * 3 * 192, device="cuda")
    chain = torch.empty(3 * (64 + 39 * 52) * 3, device="cuda")
    resid = torch.empty(3 * 39, device="cuda")

    def calls(T, o):
        t = tdm.Tiling(C=1, T=T, B=3, overlap=o, sync_every=1)
        n = t.n_maps
        tdm.ddim_run(sch, maps[:n * 4096], x0s[(T, o)], 1.0, 0.1, 0.3, 5, t, ctx=ctx)
        tdm.ddim_step(sch, 0, maps[:n * 4096], eps[:n * 4096], eps[:n * 4096], 1.0, 5, t, ctx=ctx)
        tdm.mds_recover(maps[:n * 4096], n, coords[:n * 192], ctx=ctx)
        tdm.kabsch_stitch(coords[:n * 192], t, chain[:3 * (64 + (T - 1) * (64 - o)) * 3], resid[:3 * (T - 1)],
                          ctx=ctx)

    calls(*shapes[0])
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for T, o in shapes[1:]:
        calls(T, o)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    assert tdm.ctx_sync(ctx) == 0
