"""Thin Python binding of libtdm (the tiled distance-map sampler, sm_100a).

Every function here marshals arguments to the C entry point of the same name in
``include/tdm.h`` (``ddim_run`` -> ``tdm_ddim_run`` ...) and launches on the
current torch CUDA stream.  All arithmetic runs in the library's kernels; there
is no CPU path.  Tensors must be CUDA float32, contiguous, 16-byte aligned.
PyTorch is used only for device memory and streams.

Importing the package loads ``libtdm.so`` and raises ImportError when it is
missing or stale (build it with ``python tiled_distance_maps_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtdm.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libtdm.so not found at {LIB_PATH}; build it with "
                      "`python tiled_distance_maps_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

OK, EINVAL, ECUDA, ETIMEOUT, ENONFINITE, EUNSUPPORTED, ENOMEM, ENOTCONVERGED = range(8)
STREAM_INIT, STREAM_EPS_C, STREAM_EPS_U, STREAM_ETA = range(4)
FLAG_MDS_NOT_CONVERGED = 0x1
FLAG_NONFINITE = 0x2
SCHED_COLS = 8

_c = ctypes
_vp = _c.c_void_p
_i32, _i64, _u64, _f32, _f64 = _c.c_int32, _c.c_int64, _c.c_uint64, _c.c_float, _c.c_double


class CTiling(ctypes.Structure):
    _fields_ = [("C", _i32), ("T", _i32), ("B", _i32), ("overlap", _i32), ("sync_every", _i32),
                ("reserved", _i32), ("B_total", _i64), ("b_offset", _i64), ("sample_id_base", _i64)]


_P = ctypes.POINTER
_SIGS = {
    "tdm_ctx_create": (_i32, [_P(_vp), _i32]),
    "tdm_ctx_destroy": (None, [_vp]),
    "tdm_status_str": (_c.c_char_p, [_i32]),
    "tdm_ctx_last_error": (_c.c_char_p, [_vp]),
    "tdm_ctx_sync": (_i32, [_vp, _vp, _P(_c.c_uint32)]),
    "tdm_init_schedule": (_i32, [_vp, _P(_vp), _i32, _f64, _f64, _P(_f64), _i32, _f64]),
    "tdm_schedule_destroy": (None, [_vp]),
    "tdm_schedule_table": (_i32, [_vp, _P(_f64), _i64]),
    "tdm_schedule_steps": (_i32, [_vp]),
    "tdm_init_noise": (_i32, [_vp, _vp, _P(CTiling), _u64, _vp]),
    "tdm_eps_standin": (_i32, [_vp, _vp, _i32, _vp, _vp, _f32, _i32, _u64, _P(CTiling), _vp, _vp]),
    "tdm_ddim_step": (_i32, [_vp, _vp, _i32, _vp, _vp, _vp, _f32, _u64, _P(CTiling), _vp]),
    "tdm_ddim_run": (_i32, [_vp, _vp, _vp, _vp, _f32, _f32, _f32, _u64, _i32, _P(CTiling), _vp]),
    "tdm_ddim_run_steps": (_i32, [_vp, _vp, _vp, _vp, _f32, _f32, _f32, _u64, _i32, _i32, _i32, _P(CTiling), _vp]),
    "tdm_seam_project": (_i32, [_vp, _vp, _P(CTiling), _vp]),
    "tdm_mds_recover": (_i32, [_vp, _vp, _i64, _vp, _vp, _vp]),
    "tdm_pairwise_dist": (_i32, [_vp, _vp, _i64, _vp, _vp]),
    "tdm_seam_discrepancy": (_i32, [_vp, _vp, _P(CTiling), _vp, _vp]),
    "tdm_seam_overlap_sums": (_i32, [_vp, _vp, _P(CTiling), _vp, _vp]),
    "tdm_seam_discrepancy_finalize": (_i32, [_vp, _vp, _P(CTiling), _vp, _vp]),
    "tdm_philox4x32": (_i32, [_vp, _vp, _i64, _u64, _vp, _vp]),
    "tdm_box_muller": (_i32, [_vp, _vp, _i64, _vp, _vp]),
    "tdm_seam_discrepancy_noalloc": (_i32, [_vp, _P(CTiling), _vp, _vp]),
    "tdm_kabsch_stitch": (_i32, [_vp, _vp, _P(CTiling), _vp, _vp, _vp]),
    "tdm_refine_smacof": (_i32, [_vp, _vp, _i64, _vp, _i32, _vp, _vp]),
    "tdm_nonoverlap_drift": (_i32, [_vp, _vp, _vp, _P(CTiling), _vp, _vp, _vp]),
    "tdm_cosine_alphas_bar": (_i32, [_i32, _f64, _vp]),
    "tdm_scan_nonfinite": (_i32, [_vp, _vp, _i64, _vp]),
    "tdm_fma_rate": (_i32, [_vp, ctypes.POINTER(_f64), _vp]),
    "tdm_mds_reconstruct": (_i32, [_vp, _vp, _i64, _vp, _vp, _vp, _vp]),
    "tdm_fused_lane_map": (_i32, [_i32, _i32, _vp, _i64]),
}
for _name, (_res, _args) in _SIGS.items():
    try:
        _fn = getattr(_lib, _name)
    except AttributeError as _e:
        raise ImportError(f"{LIB_PATH} does not export {_name}; rebuild it with "
                          "`python tiled_distance_maps_b200/build.py`") from _e
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


class TdmError(RuntimeError):
    def __init__(self, status: int, detail: str = ""):
        self.status = status
        msg = _lib.tdm_status_str(status).decode()
        super().__init__(f"libtdm: {msg} ({status})" + (f": {detail}" if detail else ""))


def status_str(status: int) -> str:
    return _lib.tdm_status_str(status).decode()


@dataclass
class Tiling:
    """Shape of a tiled batch ``[C][T][B][64][64]`` (see ``tdm_tiling``)."""
    C: int
    T: int
    B: int
    overlap: int = 12
    sync_every: int = 1
    B_total: int = 0
    b_offset: int = 0
    sample_id_base: int = 0

    def c(self) -> CTiling:
        return CTiling(self.C, self.T, self.B, self.overlap, self.sync_every, 0,
                       self.B_total, self.b_offset, self.sample_id_base)

    @property
    def n_maps(self) -> int:
        return self.C * self.T * self.B


class Context:
    """A libtdm context on one CUDA device (status word, scratch, plan cache)."""

    def __init__(self, device: int = 0):
        h = _vp()
        st = _lib.tdm_ctx_create(ctypes.byref(h), int(device))
        if st != OK:
            raise TdmError(st, f"tdm_ctx_create(device={device})")
        self._h = h
        self.device = int(device)

    @property
    def handle(self):
        return self._h

    def check(self, status: int):
        if status != OK:
            raise TdmError(status, _lib.tdm_ctx_last_error(self._h).decode())

    def close(self):
        if getattr(self, "_h", None):
            _lib.tdm_ctx_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


_contexts: dict[int, Context] = {}


def context(device: int | None = None) -> Context:
    """The default context of a device (created on first use)."""
    import torch
    if device is None:
        device = torch.cuda.current_device()
    ctx = _contexts.get(device)
    if ctx is None:
        ctx = _contexts[device] = Context(device)
    return ctx


class Schedule:
    """DDIM coefficient table (``tdm_init_schedule``)."""

    def __init__(self, S: int, eta: float = 0.0, T_train: int = 1000, beta_start: float = 1e-4,
                 beta_end: float = 0.02, alphas_bar=None, ctx: Context | None = None):
        self.ctx = ctx or context()
        h = _vp()
        ab = None
        if alphas_bar is not None:
            ab = (_f64 * len(alphas_bar))(*[float(v) for v in alphas_bar])
            T_train = len(alphas_bar)
        self.ctx.check(_lib.tdm_init_schedule(self.ctx.handle, ctypes.byref(h), int(T_train), float(beta_start),
                                              float(beta_end), ab, int(S), float(eta)))
        self._h = h
        self.S, self.eta, self.T_train = int(S), float(eta), int(T_train)

    @property
    def handle(self):
        return self._h

    def table(self):
        """Host float64 table ``[S][8]``: tau, ab_t, ab_p, sigma, a, b, sqrt(ab_t), 1/sqrt(1-ab_t)."""
        n = self.S * SCHED_COLS
        buf = (_f64 * n)()
        st = _lib.tdm_schedule_table(self._h, buf, n)
        if st != OK:
            raise TdmError(st)
        return [list(buf[i * SCHED_COLS:(i + 1) * SCHED_COLS]) for i in range(self.S)]

    def close(self):
        if getattr(self, "_h", None):
            _lib.tdm_schedule_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def init_schedule(S: int, eta: float = 0.0, **kw) -> Schedule:
    return Schedule(S, eta, **kw)


_torch = None
_raw_stream = None


def _t():
    """torch, imported on first use (the package imports without it)."""
    global _torch, _raw_stream
    if _torch is None:
        import torch
        _torch = torch
        # the current stream's handle without building a Stream object; the
        # public call is the fallback
        _raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    return _torch


def _ptr(t, name: str, ctx: Context | None = None):
    """Device pointer of a CUDA float32 contiguous tensor (None -> NULL)."""
    if t is None:
        return None
    torch = _t()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != torch.float32:
        raise ValueError(f"{name} must be float32, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ctx is not None and t.get_device() != ctx.device:
        raise ValueError(f"{name} is on cuda:{t.get_device()}, context on cuda:{ctx.device}")
    return _vp(t.data_ptr())


def _stream(ctx: Context):
    torch = _t()
    if _raw_stream is not None:
        return _vp(_raw_stream(ctx.device))
    return _vp(torch.cuda.current_stream(ctx.device).cuda_stream)


def _need(t, n: int, name: str):
    if t is not None and t.numel() < n:
        raise ValueError(f"{name} holds {t.numel()} floats, needs {n}")


def init_noise(maps, tiling: Tiling, seed: int, ctx: Context | None = None):
    ctx = ctx or context(maps.device.index)
    _need(maps, tiling.n_maps * 4096, "maps")
    ct = tiling.c()
    ctx.check(_lib.tdm_init_noise(ctx.handle, _ptr(maps, "maps", ctx), ctypes.byref(ct), int(seed), _stream(ctx)))
    return maps


def eps_standin(sched: Schedule, step: int, maps, x0, s: float, stream_tag: int, seed: int, tiling: Tiling,
                eps_out, ctx: Context | None = None):
    ctx = ctx or sched.ctx
    _need(maps, tiling.n_maps * 4096, "maps")
    _need(eps_out, tiling.n_maps * 4096, "eps_out")
    _need(x0, tiling.C * tiling.T * 4096, "x0")
    ct = tiling.c()
    ctx.check(_lib.tdm_eps_standin(ctx.handle, sched.handle, int(step), _ptr(maps, "maps", ctx),
                                   _ptr(x0, "x0", ctx), float(s), int(stream_tag), int(seed), ctypes.byref(ct),
                                   _ptr(eps_out, "eps_out", ctx), _stream(ctx)))
    return eps_out


def ddim_step(sched: Schedule, step: int, maps, eps_c, eps_u, w: float, seed: int, tiling: Tiling,
              ctx: Context | None = None):
    ctx = ctx or sched.ctx
    for t, nm in ((maps, "maps"), (eps_c, "eps_c"), (eps_u, "eps_u")):
        _need(t, tiling.n_maps * 4096, nm)
    ct = tiling.c()
    ctx.check(_lib.tdm_ddim_step(ctx.handle, sched.handle, int(step), _ptr(maps, "maps", ctx),
                                 _ptr(eps_c, "eps_c", ctx), _ptr(eps_u, "eps_u", ctx), float(w), int(seed),
                                 ctypes.byref(ct), _stream(ctx)))
    return maps


def ddim_run(sched: Schedule, maps, x0, w: float, s_c: float, s_u: float, seed: int, tiling: Tiling,
             init_noise: bool = True, ctx: Context | None = None, first_step: int | None = None,
             n_steps: int | None = None):
    """The fused reverse run (tdm_ddim_run); with ``first_step`` / ``n_steps``
    only that part of it (tdm_ddim_run_steps), e.g. to resume from saved maps."""
    ctx = ctx or sched.ctx
    _need(maps, tiling.n_maps * 4096, "maps")
    _need(x0, tiling.C * tiling.T * 4096, "x0")
    ct = tiling.c()
    args = (ctx.handle, sched.handle, _ptr(maps, "maps", ctx), _ptr(x0, "x0", ctx), float(w), float(s_c),
            float(s_u), int(seed), 1 if init_noise else 0)
    if first_step is None and n_steps is None:
        ctx.check(_lib.tdm_ddim_run(*args, ctypes.byref(ct), _stream(ctx)))
    else:
        first = sched.S - 1 if first_step is None else int(first_step)
        count = first + 1 if n_steps is None else int(n_steps)
        ctx.check(_lib.tdm_ddim_run_steps(*args, first, count, ctypes.byref(ct), _stream(ctx)))
    return maps


def seam_project(maps, tiling: Tiling, ctx: Context | None = None):
    ctx = ctx or context(maps.device.index)
    _need(maps, tiling.n_maps * 4096, "maps")
    ct = tiling.c()
    ctx.check(_lib.tdm_seam_project(ctx.handle, _ptr(maps, "maps", ctx), ctypes.byref(ct), _stream(ctx)))
    return maps


def mds_recover(maps, n_maps: int, coords, eigvals=None, ctx: Context | None = None):
    ctx = ctx or context(maps.device.index)
    _need(maps, n_maps * 4096, "maps")
    _need(coords, n_maps * 192, "coords")
    _need(eigvals, n_maps * 3, "eigvals")
    ctx.check(_lib.tdm_mds_recover(ctx.handle, _ptr(maps, "maps", ctx), int(n_maps), _ptr(coords, "coords", ctx),
                                   _ptr(eigvals, "eigvals", ctx), _stream(ctx)))
    return coords


def mds_reconstruct(maps, n_maps: int, coords, dist_out, eigvals=None, ctx: Context | None = None):
    """MDS recovery and the distance maps of its coordinates in one pass (see
    tdm_mds_reconstruct)."""
    ctx = ctx or context(maps.device.index)
    _need(maps, n_maps * 4096, "maps")
    _need(coords, n_maps * 192, "coords")
    _need(dist_out, n_maps * 4096, "dist_out")
    _need(eigvals, n_maps * 3, "eigvals")
    ctx.check(_lib.tdm_mds_reconstruct(ctx.handle, _ptr(maps, "maps", ctx), int(n_maps), _ptr(coords, "coords", ctx),
                                       _ptr(eigvals, "eigvals", ctx), _ptr(dist_out, "dist_out", ctx), _stream(ctx)))
    return dist_out


def pairwise_dist(coords, n_maps: int, maps_out, ctx: Context | None = None):
    ctx = ctx or context(coords.device.index)
    _need(coords, n_maps * 192, "coords")
    _need(maps_out, n_maps * 4096, "maps_out")
    ctx.check(_lib.tdm_pairwise_dist(ctx.handle, _ptr(coords, "coords", ctx), int(n_maps),
                                     _ptr(maps_out, "maps_out", ctx), _stream(ctx)))
    return maps_out


def seam_discrepancy(maps, tiling: Tiling, out, ctx: Context | None = None):
    ctx = ctx or context(maps.device.index)
    _need(maps, tiling.n_maps * 4096, "maps")
    _need(out, tiling.C * max(tiling.T - 1, 0), "out")
    ct = tiling.c()
    ctx.check(_lib.tdm_seam_discrepancy(ctx.handle, _ptr(maps, "maps", ctx), ctypes.byref(ct),
                                        _ptr(out, "out", ctx), _stream(ctx)))
    return out


def seam_overlap_sums(maps, tiling: Tiling, sums, ctx: Context | None = None):
    ctx = ctx or context(sums.device.index)
    _need(maps, tiling.n_maps * 4096, "maps")
    _need(sums, tiling.C * max(tiling.T - 1, 0) * tiling.overlap ** 2, "sums")
    ct = tiling.c()
    ctx.check(_lib.tdm_seam_overlap_sums(ctx.handle, _ptr(maps, "maps", ctx), ctypes.byref(ct),
                                         _ptr(sums, "sums", ctx), _stream(ctx)))
    return sums


def seam_discrepancy_finalize(sums, tiling: Tiling, out, ctx: Context | None = None):
    ctx = ctx or context(sums.device.index)
    _need(sums, tiling.C * max(tiling.T - 1, 0) * tiling.overlap ** 2, "sums")
    ct = tiling.c()
    ctx.check(_lib.tdm_seam_discrepancy_finalize(ctx.handle, _ptr(sums, "sums", ctx), ctypes.byref(ct),
                                                 _ptr(out, "out", ctx), _stream(ctx)))
    return out


def refine_smacof(maps, n_maps: int, coords, iterations: int, stress_out=None, ctx: Context | None = None):
    """SMACOF refinement of ``coords`` ``[n][64][3]`` (in place) against
    ``maps`` ``[n][64][64]`` (see tdm_refine_smacof)."""
    ctx = ctx or context(maps.device.index)
    _need(maps, n_maps * 4096, "maps")
    _need(coords, n_maps * 192, "coords")
    _need(stress_out, n_maps, "stress_out")
    ctx.check(_lib.tdm_refine_smacof(ctx.handle, _ptr(maps, "maps", ctx), int(n_maps), _ptr(coords, "coords", ctx),
                                     int(iterations), _ptr(stress_out, "stress_out", ctx), _stream(ctx)))
    return coords


def nonoverlap_drift(maps, ref, tiling: Tiling, tile_sums_out, drift_out=None, ctx: Context | None = None):
    """Drift of ``maps`` from ``ref`` outside the overlap blocks: per-tile
    sums ``[C][T][2]`` and optionally the per-chain ratio ``[C]`` (see
    tdm_nonoverlap_drift)."""
    ctx = ctx or context(maps.device.index)
    _need(maps, tiling.n_maps * 4096, "maps")
    _need(ref, tiling.n_maps * 4096, "ref")
    _need(tile_sums_out, tiling.C * tiling.T * 2, "tile_sums_out")
    _need(drift_out, tiling.C, "drift_out")
    ct = tiling.c()
    ctx.check(_lib.tdm_nonoverlap_drift(ctx.handle, _ptr(maps, "maps", ctx), _ptr(ref, "ref", ctx), ctypes.byref(ct),
                                        _ptr(tile_sums_out, "tile_sums_out", ctx), _ptr(drift_out, "drift_out", ctx),
                                        _stream(ctx)))
    return tile_sums_out


def cosine_alphas_bar(T_train: int = 1000, s: float = 0.008) -> list[float]:
    """The cosine alphas-bar table (Nichol & Dhariwal 2021) for
    ``Schedule(..., alphas_bar=...)`` (see tdm_cosine_alphas_bar)."""
    out = (_f64 * int(T_train))()
    st = _lib.tdm_cosine_alphas_bar(int(T_train), float(s), ctypes.cast(out, ctypes.c_void_p))
    if st != OK:
        raise TdmError(st, "cosine_alphas_bar: T_train >= 1 and s >= 0 required")
    return list(out)


def kabsch_stitch(coords, tiling: Tiling, chain_out, residual_out=None, ctx: Context | None = None):
    """Stitch per-tile coordinates ``[C][T][B][64][3]`` into chains
    ``[C][B][L][3]`` (L = 64 + (T-1)(64-overlap)); optional per-seam RMSD
    ``[C][B][T-1]`` (see tdm_kabsch_stitch)."""
    ctx = ctx or context(coords.device.index)
    L = 64 + (tiling.T - 1) * (64 - tiling.overlap)
    _need(coords, tiling.n_maps * 192, "coords")
    _need(chain_out, tiling.C * tiling.B * L * 3, "chain_out")
    _need(residual_out, tiling.C * tiling.B * max(tiling.T - 1, 0), "residual_out")
    ct = tiling.c()
    ctx.check(_lib.tdm_kabsch_stitch(ctx.handle, _ptr(coords, "coords", ctx), ctypes.byref(ct),
                                     _ptr(chain_out, "chain_out", ctx), _ptr(residual_out, "residual_out", ctx),
                                     _stream(ctx)))
    return chain_out


def seam_discrepancy_noalloc(maps, tiling: Tiling, out):
    """Eq. (6) like seam_discrepancy, for callers that cannot allocate device
    memory: no context, partial sums in the library's fixed device array (see
    tdm_seam_discrepancy_noalloc in include/tdm.h).  Runs on the current
    device and stream; calls that overlap on the GPU race on that array."""
    import torch
    _need(maps, tiling.n_maps * 4096, "maps")
    _need(out, tiling.C * max(tiling.T - 1, 0), "out")
    if out.device != maps.device:
        raise ValueError(f"out is on {out.device}, maps on {maps.device}")
    ct = tiling.c()
    # the C side runs on the current device: make it the one that holds maps
    with torch.cuda.device(maps.device):
        stream = _vp(torch.cuda.current_stream(maps.device).cuda_stream)
        st = _lib.tdm_seam_discrepancy_noalloc(_ptr(maps, "maps"), ctypes.byref(ct), _ptr(out, "out"), stream)
    if st != OK:
        raise TdmError(st, "tdm_seam_discrepancy_noalloc")
    return out


def fused_lane_map(T: int, overlap: int = 12):
    """The quad each lane of the fused run holds, as a numpy uint32 array
    ``[17 T, 32]`` of q | r << 4 | k << 10 | paired << 31 (host only; see
    tdm_fused_lane_map)."""
    import numpy as np
    out = np.empty((17 * T, 32), dtype=np.uint32)
    st = _lib.tdm_fused_lane_map(int(T), int(overlap), out.ctypes.data_as(_vp), out.size)
    if st != OK:
        raise TdmError(st, f"tdm_fused_lane_map(T={T}, overlap={overlap})")
    return out


def _uptr(t, name, ctx, dtype):
    import torch
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")
    return _vp(t.data_ptr())


def philox4x32(ctr, seed: int, out, ctx: Context | None = None):
    """out[i] = Philox4x32-10(ctr[i], seed); ctr, out: CUDA uint32 [n, 4]."""
    import torch
    ctx = ctx or context(ctr.device.index)
    n = ctr.numel() // 4
    if out.numel() < 4 * n:
        raise ValueError("out too small")
    ctx.check(_lib.tdm_philox4x32(ctx.handle, _uptr(ctr, "ctr", ctx, torch.uint32), n, int(seed),
                                  _uptr(out, "out", ctx, torch.uint32), _stream(ctx)))
    return out


def box_muller(words, z, ctx: Context | None = None):
    """z[2i], z[2i+1] from words[2i], words[2i+1]; words CUDA uint32, z float32."""
    import torch
    ctx = ctx or context(words.device.index)
    n = words.numel() // 2
    if z.numel() < 2 * n:
        raise ValueError("z too small")
    ctx.check(_lib.tdm_box_muller(ctx.handle, _uptr(words, "words", ctx, torch.uint32), n,
                                  _uptr(z, "z", ctx, torch.float32), _stream(ctx)))
    return z


def ctx_sync(ctx: Context | None = None) -> int:
    """Synchronise the current stream; return and clear the device status flags
    (FLAG_MDS_NOT_CONVERGED when an MDS eigen-solve hit its iteration cap)."""
    ctx = ctx or context()
    flags = ctypes.c_uint32(0)
    st = _lib.tdm_ctx_sync(ctx.handle, _stream(ctx), ctypes.byref(flags))
    if st not in (OK, ENOTCONVERGED, ENONFINITE):
        ctx.check(st)
    return flags.value


def scan_nonfinite(buf, ctx: Context | None = None):
    """Raise FLAG_NONFINITE (read by ctx_sync) when the float32 CUDA tensor
    ``buf`` holds NaN or inf (see tdm_scan_nonfinite)."""
    import torch
    ctx = ctx or context(buf.device.index)
    ctx.check(_lib.tdm_scan_nonfinite(ctx.handle, _uptr(buf, "buf", ctx, torch.float32), int(buf.numel()),
                                      _stream(ctx)))


def fma_rate(ctx: Context | None = None) -> float:
    """The device's measured float32 FMA rate in FMAs per second, the
    denominator of the ALU rooflines (see tdm_fma_rate); synchronises the
    current stream."""
    ctx = ctx or context()
    out = _f64(0.0)
    ctx.check(_lib.tdm_fma_rate(ctx.handle, _c.byref(out), _stream(ctx)))
    return float(out.value)
