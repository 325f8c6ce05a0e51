"""Python access to the CPU oracle (``gs_oracle.cpp``).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product (the CUDA library and its binding) never imports it, and this package
imports nothing from the product: camera records are plain objects with the
attributes listed in ``_CAM_FIELDS``.

Two precisions:
  * ``"f32"`` - the fp32 mirror: integer decisions (cull, radius, tile
    rectangle, depth-key bits, contributor counts) are taken in fp32.
  * ``"f64"`` - float64 throughout: the gradient and finite-difference
    reference.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))


class OracleCamera(ctypes.Structure):
    _fields_ = [
        ("width", ctypes.c_int), ("height", ctypes.c_int), ("tile", ctypes.c_int),
        ("fx", ctypes.c_float), ("fy", ctypes.c_float), ("cx", ctypes.c_float), ("cy", ctypes.c_float),
        ("R", ctypes.c_float * 9), ("t", ctypes.c_float * 3),
        ("z_near", ctypes.c_float), ("eps2d", ctypes.c_float), ("alpha_max", ctypes.c_float),
        ("alpha_min", ctypes.c_float), ("T_min", ctypes.c_float), ("sigma_mult", ctypes.c_float),
        ("bg", ctypes.c_float * 3),
    ]


_CAM_FIELDS = ("width", "height", "tile", "fx", "fy", "cx", "cy", "R", "t", "z_near", "eps2d",
               "alpha_max", "alpha_min", "T_min", "sigma_mult", "bg")


def camera(c) -> OracleCamera:
    oc = OracleCamera()
    oc.width, oc.height, oc.tile = int(c.width), int(c.height), int(c.tile)
    oc.fx, oc.fy, oc.cx, oc.cy = float(c.fx), float(c.fy), float(c.cx), float(c.cy)
    for k in range(9):
        oc.R[k] = float(c.R[k])
    for k in range(3):
        oc.t[k] = float(c.t[k])
        oc.bg[k] = float(c.bg[k])
    oc.z_near, oc.eps2d, oc.alpha_max = float(c.z_near), float(c.eps2d), float(c.alpha_max)
    oc.alpha_min, oc.T_min, oc.sigma_mult = float(c.alpha_min), float(c.T_min), float(c.sigma_mult)
    return oc


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        cam = ctypes.POINTER(OracleCamera)
        for suf in ("f32", "f64"):
            getattr(L, f"oracle_preprocess_{suf}").argtypes = [cam, I] + [P] * 10
            getattr(L, f"oracle_preprocess_{suf}").restype = None
            getattr(L, f"oracle_bin_{suf}").argtypes = [cam, I, P, P, P, P, P, P]
            getattr(L, f"oracle_bin_{suf}").restype = ctypes.c_longlong
            getattr(L, f"oracle_tile_list_{suf}").argtypes = [cam, I, P, P, P, I, P]
            getattr(L, f"oracle_tile_list_{suf}").restype = ctypes.c_longlong
            getattr(L, f"oracle_render_fwd_{suf}").argtypes = [cam] + [P] * 12 + [I]
            getattr(L, f"oracle_render_fwd_{suf}").restype = None
            getattr(L, f"oracle_render_bwd_{suf}").argtypes = [cam, I] + [P] * 10 + [I]
            getattr(L, f"oracle_render_bwd_{suf}").restype = None
            getattr(L, f"oracle_preprocess_bwd_{suf}").argtypes = [cam, I] + [P] * 14
            getattr(L, f"oracle_preprocess_bwd_{suf}").restype = None
        for suf, R in (("f32", ctypes.c_float), ("f64", ctypes.c_double)):
            getattr(L, f"oracle_sh_fwd_{suf}").argtypes = [cam, I, I, I, P, P, R, P]
            getattr(L, f"oracle_sh_fwd_{suf}").restype = None
            getattr(L, f"oracle_sh_bwd_{suf}").argtypes = [cam, I, I, I, P, P, R, P, P, P]
            getattr(L, f"oracle_sh_bwd_{suf}").restype = None
            getattr(L, f"oracle_sh_basis_{suf}").argtypes = [I, P, P]
            getattr(L, f"oracle_sh_basis_{suf}").restype = None
        L.oracle_exp_f32.argtypes = [P, P, ctypes.c_longlong]
        L.oracle_exp_f32.restype = None
        L.oracle_num_threads.restype = I
        L.oracle_set_threads.argtypes = [I]
        _lib = L
    return _lib


def exp_f32(x) -> np.ndarray:
    """The fp32 mirror's exp (the one its compositing uses)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty_like(x)
    lib().oracle_exp_f32(_p(x), _p(y), x.size)
    return y


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def _dt(mode: str):
    if mode == "f32":
        return np.float32
    if mode == "f64":
        return np.float64
    raise ValueError(mode)


def _a(x, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x), dtype=dtype)


def _p(x: Optional[np.ndarray]):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def preprocess(cam, means, scales, quats, opacity, mode: str = "f32") -> Dict[str, np.ndarray]:
    dt = _dt(mode)
    means, scales, quats, opacity = (_a(x, dt) for x in (means, scales, quats, opacity))
    n = means.shape[0]
    out = dict(mean2d=np.zeros((n, 2), dt), depth=np.zeros(n, dt), conic_opacity=np.zeros((n, 4), dt),
               radius=np.zeros(n, np.int32), rect=np.zeros((n, 4), np.int32),
               tiles_touched=np.zeros(n, np.uint32))
    oc = camera(cam)
    getattr(lib(), f"oracle_preprocess_{mode}")(
        ctypes.byref(oc), n, _p(means), _p(scales), _p(quats), _p(opacity), _p(out["mean2d"]), _p(out["depth"]),
        _p(out["conic_opacity"]), _p(out["radius"]), _p(out["rect"]), _p(out["tiles_touched"]))
    return out


def bin_pairs(cam, depth, rect, tiles_touched, mode: str = "f32", want_keys: bool = True) -> Dict[str, np.ndarray]:
    """Every (tile, Gaussian) pair in (tile, depth, id) order: ``ids`` [P],
    ``ranges`` [T, 2] and, with ``want_keys``, the 64-bit (tile << 32 | depth
    bits) keys."""
    dt = _dt(mode)
    depth = _a(depth, dt)
    rect = _a(rect, np.int32)
    tt = _a(tiles_touched, np.uint32)
    P = int(tt.astype(np.uint64).sum())
    keys = np.zeros(P, np.uint64) if want_keys else None
    ids = np.zeros(P, np.uint32)
    ranges = np.zeros((cam.tiles_x * cam.tiles_y if hasattr(cam, "tiles_x") else
                       ((cam.width + cam.tile - 1) // cam.tile) * ((cam.height + cam.tile - 1) // cam.tile), 2),
                      np.uint32)
    oc = camera(cam)
    got = getattr(lib(), f"oracle_bin_{mode}")(ctypes.byref(oc), depth.shape[0], _p(depth), _p(rect), _p(tt),
                                                _p(keys), _p(ids), _p(ranges))
    assert got == P
    return dict(keys=keys, ids=ids, ranges=ranges, num_pairs=P)


def tile_list(cam, depth, rect, tiles_touched, tile: int, mode: str = "f32") -> np.ndarray:
    dt = _dt(mode)
    depth = _a(depth, dt)
    rect = _a(rect, np.int32)
    tt = _a(tiles_touched, np.uint32)
    oc = camera(cam)
    fn = getattr(lib(), f"oracle_tile_list_{mode}")
    n = fn(ctypes.byref(oc), depth.shape[0], _p(depth), _p(rect), _p(tt), int(tile), None)
    out = np.zeros(n, np.uint32)
    fn(ctypes.byref(oc), depth.shape[0], _p(depth), _p(rect), _p(tt), int(tile), _p(out))
    return out


def render_fwd(cam, ranges, ids, mean2d, conic_opacity, colors, mode: str = "f32",
               tiles: Optional[Sequence[int]] = None, blend_mask: bool = False) -> Dict[str, np.ndarray]:
    """Compositing forward.  With ``blend_mask``, also the per-quadrant mask:
    for sorted position k and 8x8 quadrant q of k's tile, bit (k & 31) of
    word (k >> 5) * 4 + q is set when that term was blended into a pixel of
    the quadrant."""
    dt = _dt(mode)
    ranges = _a(ranges, np.uint32)
    ids = _a(ids, np.uint32)
    mean2d, conic_opacity, colors = (_a(x, dt) for x in (mean2d, conic_opacity, colors))
    H, W = cam.height, cam.width
    out = dict(image=np.zeros((3, H, W), dt), final_T=np.zeros((H, W), dt),
               n_contrib=np.zeros((H, W), np.uint32), n_eval=np.zeros((H, W), np.uint32),
               n_blended=np.zeros((H, W), np.uint32))
    if blend_mask:
        out["blend_mask"] = np.zeros(4 * ((ids.size + 31) // 32), np.uint32)
    sub = None if tiles is None else _a(tiles, np.int32)
    oc = camera(cam)
    getattr(lib(), f"oracle_render_fwd_{mode}")(
        ctypes.byref(oc), _p(ranges), _p(ids), _p(mean2d), _p(conic_opacity), _p(colors), _p(out["image"]),
        _p(out["final_T"]), _p(out["n_contrib"]), _p(out["n_eval"]), _p(out["n_blended"]),
        _p(out.get("blend_mask")), _p(sub), 0 if sub is None else sub.size)
    return out


def render_bwd(cam, N: int, ranges, ids, mean2d, conic_opacity, colors, dL_dimage, mode: str = "f64",
               tiles: Optional[Sequence[int]] = None) -> Dict[str, np.ndarray]:
    dt = _dt(mode)
    ranges = _a(ranges, np.uint32)
    ids = _a(ids, np.uint32)
    mean2d, conic_opacity, colors, dL_dimage = (_a(x, dt) for x in (mean2d, conic_opacity, colors, dL_dimage))
    out = dict(dL_dmean2d=np.zeros((N, 2), dt), dL_dconic_opacity=np.zeros((N, 4), dt),
               dL_dcolor=np.zeros((N, 3), dt))
    sub = None if tiles is None else _a(tiles, np.int32)
    oc = camera(cam)
    getattr(lib(), f"oracle_render_bwd_{mode}")(
        ctypes.byref(oc), int(N), _p(ranges), _p(ids), _p(mean2d), _p(conic_opacity), _p(colors), _p(dL_dimage),
        _p(out["dL_dmean2d"]), _p(out["dL_dconic_opacity"]), _p(out["dL_dcolor"]), _p(sub),
        0 if sub is None else sub.size)
    return out


def preprocess_bwd(cam, means, scales, quats, radius, dL_dmean2d, dL_dconic_opacity, dL_dcolor2d,
                   mode: str = "f64", accumulate_into: Optional[Dict[str, np.ndarray]] = None,
                   densify: bool = False) -> Dict[str, np.ndarray]:
    dt = _dt(mode)
    means, scales, quats = (_a(x, dt) for x in (means, scales, quats))
    radius = _a(radius, np.int32)
    dm, dc, dcol = (_a(x, dt) for x in (dL_dmean2d, dL_dconic_opacity, dL_dcolor2d))
    n = means.shape[0]
    out = accumulate_into or dict(dL_dmeans=np.zeros((n, 3), dt), dL_dscales=np.zeros((n, 3), dt),
                                  dL_dquats=np.zeros((n, 4), dt), dL_dopacity=np.zeros(n, dt),
                                  dL_dcolors=np.zeros((n, 3), dt))
    if densify and "grad2d_accum" not in out:
        out["grad2d_accum"] = np.zeros(n, dt)
        out["vis_count"] = np.zeros(n, np.uint32)
    oc = camera(cam)
    getattr(lib(), f"oracle_preprocess_bwd_{mode}")(
        ctypes.byref(oc), n, _p(means), _p(scales), _p(quats), _p(radius), _p(dm), _p(dc), _p(dcol),
        _p(out["dL_dmeans"]), _p(out["dL_dscales"]), _p(out["dL_dquats"]), _p(out["dL_dopacity"]),
        _p(out["dL_dcolors"]), _p(out.get("grad2d_accum")), _p(out.get("vis_count")))
    return out


def forward(cam, means, scales, quats, opacity, colors, mode: str = "f64",
            tiles: Optional[Sequence[int]] = None) -> Dict[str, np.ndarray]:
    """Preprocess, binning and compositing for one camera (compositing of
    the listed ``tiles`` only, when given)."""
    pre = preprocess(cam, means, scales, quats, opacity, mode)
    b = bin_pairs(cam, pre["depth"], pre["rect"], pre["tiles_touched"], mode, want_keys=False)
    r = render_fwd(cam, b["ranges"], b["ids"], pre["mean2d"], pre["conic_opacity"], colors, mode, tiles=tiles)
    return dict(pre=pre, bins=b, **r)


def forward_backward(cam, means, scales, quats, opacity, colors, dL_dimage, mode: str = "f64"
                     ) -> Dict[str, np.ndarray]:
    """The whole path for one camera: forward, then the gradient of
    L = sum(dL_dimage * image) w.r.t. means, scales, quats, opacity, colours."""
    f = forward(cam, means, scales, quats, opacity, colors, mode)
    pre, b = f["pre"], f["bins"]
    g2 = render_bwd(cam, np.asarray(means).shape[0], b["ranges"], b["ids"], pre["mean2d"], pre["conic_opacity"],
                    colors, dL_dimage, mode)
    g3 = preprocess_bwd(cam, means, scales, quats, pre["radius"], g2["dL_dmean2d"], g2["dL_dconic_opacity"],
                        g2["dL_dcolor"], mode)
    f.update(g2)
    f.update(g3)
    return f


# --------------------------------------------------------------------------
# Spherical-harmonics colour
# --------------------------------------------------------------------------

def sh_basis(dirs, mode: str = "f64") -> np.ndarray:
    """The 16 real SH basis values (degree <= 3) at unit directions [n, 3]."""
    dt = _dt(mode)
    d = _a(dirs, dt).reshape(-1, 3)
    out = np.zeros((d.shape[0], 16), dt)
    getattr(lib(), f"oracle_sh_basis_{mode}")(d.shape[0], _p(d), _p(out))
    return out


def sh_fwd(cam, means, sh, degree: int, offset: float = 0.0, mode: str = "f64") -> np.ndarray:
    dt = _dt(mode)
    means, sh = _a(means, dt), _a(sh, dt)
    n, K = means.shape[0], sh.shape[1]
    out = np.zeros((n, 3), dt)
    oc = camera(cam)
    getattr(lib(), f"oracle_sh_fwd_{mode}")(ctypes.byref(oc), n, int(degree), K, _p(means), _p(sh), float(offset),
                                            _p(out))
    return out


def sh_bwd(cam, means, sh, degree: int, dL_dcolors, offset: float = 0.0, mode: str = "f64",
           accumulate_into: Optional[Dict[str, np.ndarray]] = None) -> Dict[str, np.ndarray]:
    dt = _dt(mode)
    means, sh, g = _a(means, dt), _a(sh, dt), _a(dL_dcolors, dt)
    n, K = means.shape[0], sh.shape[1]
    out = accumulate_into or dict(dL_dsh=np.zeros_like(sh), dL_dmeans=np.zeros_like(means))
    oc = camera(cam)
    getattr(lib(), f"oracle_sh_bwd_{mode}")(ctypes.byref(oc), n, int(degree), K, _p(means), _p(sh), float(offset),
                                            _p(g), _p(out["dL_dsh"]), _p(out["dL_dmeans"]))
    return out
