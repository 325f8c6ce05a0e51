"""Thin Python binding of ``libgs.so`` (the C ABI declared in ``include/gs.h``).

Argument marshalling only: every function here checks the tensors it is given
(device, dtype, shape, contiguity), passes raw device pointers and the current
CUDA stream to the C entry point of the same name, and raises on a non-zero
status.  All arithmetic runs in the library's CUDA kernels.  There is no CPU
path: if ``libgs.so`` is missing or no CUDA device is present, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# GS_LIBRARY=debug loads libgs_debug.so (the index-checking build); any other
# value is taken as a path to the library.
_choice = os.environ.get("GS_LIBRARY", "")
LIB_PATH = (os.path.join(_HERE, "libgs_debug.so") if _choice == "debug" else
            (_choice or os.path.join(_HERE, "libgs.so")))

GS_OK = 0
GS_ERR_INVALID_ARG = 1
GS_ERR_CAPACITY = 2
GS_ERR_TIMEOUT = 4
GS_ERR_CUDA = 8
GS_ERR_UNIMPLEMENTED = 16
GS_ERR_OVERFLOW = 32
GS_ERR_INDEX = 64
GS_STAGE_PREPROCESS_FWD = 0
GS_STAGE_BIN_SORT = 1
TILE = 16

# Every symbol include/gs.h declares.
EXPORTED = ("gs_version", "gs_launch_count", "gs_status_string", "gs_workspace_bytes", "gs_read_status", "gs_clear_status",
            "gs_preprocess_fwd", "gs_bin_sort", "gs_render_fwd", "gs_render_bwd", "gs_preprocess_bwd",
            "gs_preprocess_fwd_noalloc", "gs_render_stats", "gs_sh_fwd", "gs_sh_bwd", "gs_sh_fwd_f16",
            "gs_sh_bwd_f16", "gs_adam_step", "gs_debug_configure", "gs_debug_read")


class GsCamera(ctypes.Structure):
    """Mirror of ``gs_camera`` in include/gs.h."""
    _fields_ = [
        ("width", ctypes.c_int), ("height", ctypes.c_int), ("tile", ctypes.c_int),
        ("fx", ctypes.c_float), ("fy", ctypes.c_float), ("cx", ctypes.c_float), ("cy", ctypes.c_float),
        ("R", ctypes.c_float * 9), ("t", ctypes.c_float * 3),
        ("z_near", ctypes.c_float), ("eps2d", ctypes.c_float), ("alpha_max", ctypes.c_float),
        ("alpha_min", ctypes.c_float), ("T_min", ctypes.c_float), ("sigma_mult", ctypes.c_float),
        ("bg", ctypes.c_float * 3),
    ]


class GsAdamConfig(ctypes.Structure):
    """gs_adam_config: per-group learning rates, Adam's betas and eps, and the
    warm-up length of the position and scale rates."""
    _fields_ = [("lr_means", ctypes.c_float), ("lr_scales", ctypes.c_float), ("lr_quats", ctypes.c_float),
                ("lr_opacity", ctypes.c_float), ("lr_colors", ctypes.c_float), ("beta1", ctypes.c_float),
                ("beta2", ctypes.c_float), ("eps", ctypes.c_float), ("warmup_steps", ctypes.c_int)]


class GsError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: status {status} ({status_string(status)})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libgs.so; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "differentiable_gaussian_splatting_preprocess_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I, U, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
        cam = ctypes.POINTER(GsCamera)
        L.gs_version.restype = I
        L.gs_version.argtypes = []
        L.gs_launch_count.restype = ctypes.c_ulonglong
        L.gs_launch_count.argtypes = []
        L.gs_status_string.restype = ctypes.c_char_p
        L.gs_status_string.argtypes = [I]
        L.gs_workspace_bytes.restype = S
        L.gs_workspace_bytes.argtypes = [I, I, U, I, I]
        L.gs_read_status.restype = I
        L.gs_read_status.argtypes = [P, ctypes.POINTER(I), P]
        L.gs_clear_status.restype = I
        L.gs_clear_status.argtypes = [P, P]
        L.gs_preprocess_fwd.restype = I
        L.gs_preprocess_fwd.argtypes = [cam, I] + [P] * 11 + [P, S, P]
        L.gs_bin_sort.restype = I
        L.gs_bin_sort.argtypes = [cam, I, P, P, P, P, U, P, P, P, P, S, P]
        L.gs_render_fwd.restype = I
        L.gs_render_fwd.argtypes = [cam] + [P] * 9 + [U, P]
        L.gs_render_stats.restype = I
        L.gs_render_stats.argtypes = [cam] + [P] * 6 + [P]
        L.gs_render_bwd.restype = I
        L.gs_render_bwd.argtypes = [cam, I] + [P] * 8 + [U] + [P] * 4 + [P]
        L.gs_sh_fwd.restype = I
        L.gs_sh_fwd.argtypes = [cam, I, I, I, P, P, ctypes.c_float, P, P]
        L.gs_sh_bwd.restype = I
        L.gs_sh_bwd.argtypes = [cam, I, I, I, P, P, ctypes.c_float, P, P, P, P]
        L.gs_preprocess_fwd_noalloc.restype = I
        L.gs_preprocess_fwd_noalloc.argtypes = [cam, I] + [P] * 11 + [P]
        L.gs_adam_step.restype = I
        L.gs_adam_step.argtypes = [ctypes.POINTER(GsAdamConfig), I, I, I] + [P] * 14 + [P]
        L.gs_sh_fwd_f16.restype = I
        L.gs_sh_fwd_f16.argtypes = [cam, I, I, I, P, P, ctypes.c_float, P, P]
        L.gs_sh_bwd_f16.restype = I
        L.gs_sh_bwd_f16.argtypes = [cam, I, I, I, P, P, ctypes.c_float, P, P, P, P]
        L.gs_preprocess_bwd.restype = I
        L.gs_preprocess_bwd.argtypes = [cam, I] + [P] * 15 + [P]
        L.gs_debug_configure.restype = I
        L.gs_debug_configure.argtypes = [U, U]
        L.gs_debug_read.restype = I
        L.gs_debug_read.argtypes = [ctypes.POINTER(I), I]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gs_status_string(int(status)).decode()


def version() -> int:
    return int(lib().gs_version())


def launch_count() -> int:
    """Kernels the library has launched in this process so far."""
    return int(lib().gs_launch_count())


def camera_struct(cam) -> GsCamera:
    """Build the C camera record from any object with the gs_camera fields."""
    c = GsCamera()
    c.width, c.height, c.tile = int(cam.width), int(cam.height), int(getattr(cam, "tile", TILE))
    c.fx, c.fy, c.cx, c.cy = float(cam.fx), float(cam.fy), float(cam.cx), float(cam.cy)
    for k in range(9):
        c.R[k] = float(cam.R[k])
    for k in range(3):
        c.t[k] = float(cam.t[k])
        c.bg[k] = float(cam.bg[k])
    c.z_near, c.eps2d, c.alpha_max = float(cam.z_near), float(cam.eps2d), float(cam.alpha_max)
    c.alpha_min, c.T_min, c.sigma_mult = float(cam.alpha_min), float(cam.T_min), float(cam.sigma_mult)
    return c


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[ctypes.c_void_p]:
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t: Optional[torch.Tensor], name: str, dtype, shape=None, optional: bool = False) -> None:
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _ok(fn: str, status: int) -> None:
    if status != GS_OK:
        raise GsError(fn, status)


def num_tiles(cam) -> int:
    return ((cam.width + TILE - 1) // TILE) * ((cam.height + TILE - 1) // TILE)


def gs_debug_configure(n_gauss: int, capacity: int) -> None:
    """Debug build only: the limits of its index checks (Gaussian ids below
    n_gauss, list positions below capacity); clears the debug word."""
    _ok("gs_debug_configure", lib().gs_debug_configure(int(n_gauss), int(capacity)))


def gs_debug_read(clear: bool = False) -> int:
    """Debug build only: the debug word (GS_ERR_INDEX once a check failed);
    waits for the device."""
    f = ctypes.c_int(0)
    _ok("gs_debug_read", lib().gs_debug_read(ctypes.byref(f), 1 if clear else 0))
    return int(f.value)


def gs_workspace_bytes(stage: int, N: int, capacity: int, width: int, height: int) -> int:
    return int(lib().gs_workspace_bytes(int(stage), int(N), int(capacity), int(width), int(height)))


def gs_read_status(ws: torch.Tensor, stream=None) -> int:
    st = ctypes.c_int(0)
    _ok("gs_read_status", lib().gs_read_status(_ptr(ws), ctypes.byref(st), _stream(stream)))
    return int(st.value)


def gs_clear_status(ws: torch.Tensor, stream=None) -> None:
    _ok("gs_clear_status", lib().gs_clear_status(_ptr(ws), _stream(stream)))


def gs_preprocess_fwd(cam, means, scales, quats, opacity, mean2d, depth, conic_opacity, radius, rect,
                      tiles_touched, d_num_pairs, ws, stream=None) -> None:
    N = means.shape[0]
    f32, i32, u32 = torch.float32, torch.int32, torch.uint32
    _check(means, "means", f32, (N, 3))
    _check(scales, "scales", f32, (N, 3))
    _check(quats, "quats", f32, (N, 4))
    _check(opacity, "opacity", f32, (N,))
    _check(mean2d, "mean2d", f32, (N, 2))
    _check(depth, "depth", f32, (N,))
    _check(conic_opacity, "conic_opacity", f32, (N, 4))
    _check(radius, "radius", i32, (N,))
    _check(rect, "rect", i32, (N, 4))
    _check(tiles_touched, "tiles_touched", u32, (N,))
    _check(d_num_pairs, "d_num_pairs", u32)
    _check(ws, "ws", torch.uint8)
    c = camera_struct(cam)
    _ok("gs_preprocess_fwd", lib().gs_preprocess_fwd(
        ctypes.byref(c), int(N), _ptr(means), _ptr(scales), _ptr(quats), _ptr(opacity), _ptr(mean2d), _ptr(depth),
        _ptr(conic_opacity), _ptr(radius), _ptr(rect), _ptr(tiles_touched), _ptr(d_num_pairs), _ptr(ws),
        ws.numel(), _stream(stream)))


def gs_bin_sort(cam, depth, rect, tiles_touched, d_num_pairs, capacity: int, ids, ranges, keys, ws,
                stream=None) -> None:
    N = depth.shape[0]
    _check(depth, "depth", torch.float32, (N,))
    _check(rect, "rect", torch.int32, (N, 4))
    _check(tiles_touched, "tiles_touched", torch.uint32, (N,))
    _check(d_num_pairs, "d_num_pairs", torch.uint32)
    _check(ids, "ids", torch.uint32)
    if ids.numel() < capacity:
        raise ValueError("ids holds fewer elements than capacity")
    _check(ranges, "ranges", torch.uint32, (num_tiles(cam), 2))
    _check(keys, "keys", torch.uint64, optional=True)
    if keys is not None and keys.numel() < capacity:
        raise ValueError("keys holds fewer elements than capacity")
    _check(ws, "ws", torch.uint8)
    c = camera_struct(cam)
    _ok("gs_bin_sort", lib().gs_bin_sort(
        ctypes.byref(c), int(N), _ptr(depth), _ptr(rect), _ptr(tiles_touched), _ptr(d_num_pairs), int(capacity),
        _ptr(ids), _ptr(ranges), _ptr(keys), _ptr(ws), ws.numel(), _stream(stream)))


def order_words(n_tiles: int) -> int:
    """Words of the dispatch-order block at the start of the contribution
    mask (GS_ORDER_WORDS): per quadrant its blended-position count and the
    backward's dispatch order, per tile the forward's dispatch order, and
    the per-partition class counts of the quadrants."""
    return 12 * int(n_tiles) + 256


def mask_words(capacity: int, n_tiles: int) -> int:
    """Words of the contribution mask (GS_MASK_WORDS) for `capacity` sorted
    pairs on an image of `n_tiles` tiles: the dispatch-order block, then the
    contribution bits."""
    return order_words(n_tiles) + 4 * ((int(capacity) + 31) // 32)


def _check_mask(cam, contrib_mask) -> None:
    _check(contrib_mask, "contrib_mask", torch.uint32, optional=True)
    if contrib_mask is not None and (contrib_mask.numel() < order_words(num_tiles(cam)) + 4
                                     or contrib_mask.numel() % 4):
        raise ValueError("contrib_mask needs a multiple of 4 words, at least mask_words(1, num_tiles(cam))")


def gs_render_fwd(cam, ranges, ids, mean2d, conic_opacity, colors, image, final_T, n_contrib, contrib_mask=None,
                  stream=None) -> None:
    N = mean2d.shape[0]
    H, W = cam.height, cam.width
    _check(ranges, "ranges", torch.uint32, (num_tiles(cam), 2))
    _check(ids, "ids", torch.uint32)
    _check(mean2d, "mean2d", torch.float32, (N, 2))
    _check(conic_opacity, "conic_opacity", torch.float32, (N, 4))
    _check(colors, "colors", torch.float32, (N, 3))
    _check(image, "image", torch.float32, (3, H, W))
    _check(final_T, "final_T", torch.float32, (H, W))
    _check(n_contrib, "n_contrib", torch.uint32, (H, W))
    _check_mask(cam, contrib_mask)
    c = camera_struct(cam)
    _ok("gs_render_fwd", lib().gs_render_fwd(
        ctypes.byref(c), _ptr(ranges), _ptr(ids), _ptr(mean2d), _ptr(conic_opacity), _ptr(colors), _ptr(image),
        _ptr(final_T), _ptr(n_contrib), _ptr(contrib_mask), 0 if contrib_mask is None else contrib_mask.numel(),
        _stream(stream)))


def gs_render_stats(cam, ranges, ids, mean2d, conic_opacity, n_evaluated, n_blended, stream=None) -> None:
    N = mean2d.shape[0]
    H, W = cam.height, cam.width
    _check(ranges, "ranges", torch.uint32, (num_tiles(cam), 2))
    _check(ids, "ids", torch.uint32)
    _check(mean2d, "mean2d", torch.float32, (N, 2))
    _check(conic_opacity, "conic_opacity", torch.float32, (N, 4))
    _check(n_evaluated, "n_evaluated", torch.uint32, (H, W))
    _check(n_blended, "n_blended", torch.uint32, (H, W))
    c = camera_struct(cam)
    _ok("gs_render_stats", lib().gs_render_stats(
        ctypes.byref(c), _ptr(ranges), _ptr(ids), _ptr(mean2d), _ptr(conic_opacity), _ptr(n_evaluated),
        _ptr(n_blended), _stream(stream)))


def gs_render_bwd(cam, ranges, ids, mean2d, conic_opacity, colors, final_T, n_contrib, dL_dimage, dL_dmean2d,
                  dL_dconic_opacity, dL_dcolor, contrib_mask=None, stream=None) -> None:
    N = mean2d.shape[0]
    H, W = cam.height, cam.width
    _check(ranges, "ranges", torch.uint32, (num_tiles(cam), 2))
    _check(ids, "ids", torch.uint32)
    _check(mean2d, "mean2d", torch.float32, (N, 2))
    _check(conic_opacity, "conic_opacity", torch.float32, (N, 4))
    _check(colors, "colors", torch.float32, (N, 3))
    _check(final_T, "final_T", torch.float32, (H, W))
    _check(n_contrib, "n_contrib", torch.uint32, (H, W))
    _check(dL_dimage, "dL_dimage", torch.float32, (3, H, W))
    _check(dL_dmean2d, "dL_dmean2d", torch.float32, (N, 2))
    _check(dL_dconic_opacity, "dL_dconic_opacity", torch.float32, (N, 4))
    _check(dL_dcolor, "dL_dcolor", torch.float32, (N, 3))
    _check_mask(cam, contrib_mask)
    c = camera_struct(cam)
    _ok("gs_render_bwd", lib().gs_render_bwd(
        ctypes.byref(c), int(N), _ptr(ranges), _ptr(ids), _ptr(mean2d), _ptr(conic_opacity), _ptr(colors),
        _ptr(final_T), _ptr(n_contrib), _ptr(contrib_mask), 0 if contrib_mask is None else contrib_mask.numel(),
        _ptr(dL_dimage), _ptr(dL_dmean2d), _ptr(dL_dconic_opacity), _ptr(dL_dcolor), _stream(stream)))


def gs_preprocess_bwd(cam, means, scales, quats, radius, conic_opacity, dL_dmean2d, dL_dconic_opacity,
                      dL_dcolor2d, dL_dmeans, dL_dscales, dL_dquats, dL_dopacity, dL_dcolors, grad2d_accum=None,
                      vis_count=None, stream=None) -> None:
    N = means.shape[0]
    f32 = torch.float32
    _check(means, "means", f32, (N, 3))
    _check(scales, "scales", f32, (N, 3))
    _check(quats, "quats", f32, (N, 4))
    _check(radius, "radius", torch.int32, (N,))
    _check(conic_opacity, "conic_opacity", f32, (N, 4))
    _check(dL_dmean2d, "dL_dmean2d", f32, (N, 2))
    _check(dL_dconic_opacity, "dL_dconic_opacity", f32, (N, 4))
    _check(dL_dcolor2d, "dL_dcolor2d", f32, (N, 3))
    _check(dL_dmeans, "dL_dmeans", f32, (N, 3))
    _check(dL_dscales, "dL_dscales", f32, (N, 3))
    _check(dL_dquats, "dL_dquats", f32, (N, 4))
    _check(dL_dopacity, "dL_dopacity", f32, (N,))
    _check(dL_dcolors, "dL_dcolors", f32, (N, 3))
    _check(grad2d_accum, "grad2d_accum", f32, (N,), optional=True)
    _check(vis_count, "vis_count", torch.uint32, (N,), optional=True)
    c = camera_struct(cam)
    _ok("gs_preprocess_bwd", lib().gs_preprocess_bwd(
        ctypes.byref(c), int(N), _ptr(means), _ptr(scales), _ptr(quats), _ptr(radius), _ptr(conic_opacity),
        _ptr(dL_dmean2d), _ptr(dL_dconic_opacity), _ptr(dL_dcolor2d), _ptr(dL_dmeans), _ptr(dL_dscales),
        _ptr(dL_dquats), _ptr(dL_dopacity), _ptr(dL_dcolors), _ptr(grad2d_accum), _ptr(vis_count),
        _stream(stream)))


NOALLOC_MAX_GAUSSIANS = 1 << 24
SH_MAX_DEGREE = 3


def _sh_entry(name: str, sh):
    """The fp32 entry point, or its half-precision-storage twin for float16
    coefficients."""
    if sh.dtype == torch.float16:
        return name + "_f16"
    _check(sh, "sh", torch.float32)
    return name


def gs_sh_fwd(cam, degree: int, means, sh, colors, offset: float = 0.0, stream=None) -> None:
    """SH colour; `sh` [N, K, 3] float32, or float16 (storage only: the
    kernel computes in fp32)."""
    N = means.shape[0]
    _check(means, "means", torch.float32, (N, 3))
    name = _sh_entry("gs_sh_fwd", sh)
    _check(sh, "sh", sh.dtype)
    if sh.dim() != 3 or sh.shape[0] != N or sh.shape[2] != 3:
        raise ValueError("sh must have shape [N, K, 3]")
    _check(colors, "colors", torch.float32, (N, 3))
    c = camera_struct(cam)
    _ok(name, getattr(lib(), name)(ctypes.byref(c), int(N), int(degree), int(sh.shape[1]), _ptr(means), _ptr(sh),
                                   float(offset), _ptr(colors), _stream(stream)))


def gs_sh_bwd(cam, degree: int, means, sh, dL_dcolors, dL_dsh, dL_dmeans, offset: float = 0.0, stream=None) -> None:
    """SH backward; `sh` float32 or float16 (storage only); dL_dsh is float32
    [N, K, 3] in both cases and is accumulated into."""
    N = means.shape[0]
    _check(means, "means", torch.float32, (N, 3))
    name = _sh_entry("gs_sh_bwd", sh)
    _check(sh, "sh", sh.dtype)
    if sh.dim() != 3 or sh.shape[0] != N or sh.shape[2] != 3:
        raise ValueError("sh must have shape [N, K, 3]")
    _check(dL_dcolors, "dL_dcolors", torch.float32, (N, 3))
    _check(dL_dsh, "dL_dsh", torch.float32, tuple(sh.shape))
    _check(dL_dmeans, "dL_dmeans", torch.float32, (N, 3))
    c = camera_struct(cam)
    _ok(name, getattr(lib(), name)(ctypes.byref(c), int(N), int(degree), int(sh.shape[1]), _ptr(means), _ptr(sh),
                                   float(offset), _ptr(dL_dcolors), _ptr(dL_dsh), _ptr(dL_dmeans),
                                   _stream(stream)))


def gs_sh_fwd_f16(cam, degree: int, means, sh, colors, offset: float = 0.0, stream=None) -> None:
    if sh.dtype != torch.float16:
        raise TypeError("gs_sh_fwd_f16 takes float16 coefficients")
    gs_sh_fwd(cam, degree, means, sh, colors, offset, stream)


def gs_sh_bwd_f16(cam, degree: int, means, sh, dL_dcolors, dL_dsh, dL_dmeans, offset: float = 0.0,
                  stream=None) -> None:
    if sh.dtype != torch.float16:
        raise TypeError("gs_sh_bwd_f16 takes float16 coefficients")
    gs_sh_bwd(cam, degree, means, sh, dL_dcolors, dL_dsh, dL_dmeans, offset, stream)


def gs_preprocess_fwd_noalloc(cam, means, scales, quats, opacity, mean2d, depth, conic_opacity, radius, rect,
                              tiles_touched, d_num_pairs, stream=None) -> None:
    """gs_preprocess_fwd without a workspace, for callers that cannot
    allocate device memory: the scratch is a fixed array inside libgs.so
    (N up to NOALLOC_MAX_GAUSSIANS; calls on one device must not overlap)."""
    fn = lib().gs_preprocess_fwd_noalloc
    N = means.shape[0]
    f32, i32, u32 = torch.float32, torch.int32, torch.uint32
    _check(means, "means", f32, (N, 3))
    _check(scales, "scales", f32, (N, 3))
    _check(quats, "quats", f32, (N, 4))
    _check(opacity, "opacity", f32, (N,))
    _check(mean2d, "mean2d", f32, (N, 2))
    _check(depth, "depth", f32, (N,))
    _check(conic_opacity, "conic_opacity", f32, (N, 4))
    _check(radius, "radius", i32, (N,))
    _check(rect, "rect", i32, (N, 4))
    _check(tiles_touched, "tiles_touched", u32, (N,))
    _check(d_num_pairs, "d_num_pairs", u32)
    c = camera_struct(cam)
    _ok("gs_preprocess_fwd_noalloc", fn(
        ctypes.byref(c), int(N), _ptr(means), _ptr(scales), _ptr(quats), _ptr(opacity), _ptr(mean2d), _ptr(depth),
        _ptr(conic_opacity), _ptr(radius), _ptr(rect), _ptr(tiles_touched), _ptr(d_num_pairs), _stream(stream)))


def gs_adam_step(cfg: GsAdamConfig, step: int, params: dict, grads: dict, m, v, scales=None, opacity=None,
                 stream=None) -> None:
    """Fused Adam step.  ``params``: means [N,3], log_scales [N,3], quats [N,4],
    logit_opacity [N], colors [N,C] (float32, updated in place); ``grads``:
    dL_dmeans, dL_dscales, dL_dquats, dL_dopacity, dL_dcolors as returned by
    the rasterizer (w.r.t. activated scales and opacity); ``m``, ``v``: float32
    [(11 + C) N] moments (zero before step 1); ``scales``, ``opacity``:
    optional outputs of the new activated values."""
    N = params["means"].shape[0]
    colors = params["colors"]
    C = colors.shape[1] if colors.dim() == 2 else int(colors[0].numel()) if N else 0
    f32 = torch.float32
    for k, shp in (("means", (N, 3)), ("log_scales", (N, 3)), ("quats", (N, 4)), ("logit_opacity", (N,))):
        _check(params[k], k, f32, shp)
    _check(colors, "colors", f32)
    for k, shp in (("dL_dmeans", (N, 3)), ("dL_dscales", (N, 3)), ("dL_dquats", (N, 4)), ("dL_dopacity", (N,))):
        _check(grads[k], k, f32, shp)
    _check(grads["dL_dcolors"], "dL_dcolors", f32, tuple(colors.shape))
    _check(m, "m", f32, ((11 + C) * N,))
    _check(v, "v", f32, ((11 + C) * N,))
    _check(scales, "scales", f32, (N, 3), optional=True)
    _check(opacity, "opacity", f32, (N,), optional=True)
    _ok("gs_adam_step", lib().gs_adam_step(
        ctypes.byref(cfg), int(step), int(N), int(C), _ptr(params["means"]), _ptr(params["log_scales"]),
        _ptr(params["quats"]), _ptr(params["logit_opacity"]), _ptr(colors), _ptr(grads["dL_dmeans"]),
        _ptr(grads["dL_dscales"]), _ptr(grads["dL_dquats"]), _ptr(grads["dL_dopacity"]), _ptr(grads["dL_dcolors"]),
        _ptr(m), _ptr(v), _ptr(scales), _ptr(opacity), _stream(stream)))
