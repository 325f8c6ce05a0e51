"""Seeded synthetic scenes for the Gaussian-splatting rasterizer.

This module only draws inputs.  It contains none of the rasterizer's
arithmetic: no projection, no covariance, no compositing.  Both the CUDA path
and the CPU oracle consume the arrays it returns, so it is the one module the
two sides share.

Every scene is drawn with numpy's PCG64 generator (seed 0 unless stated) in a
fixed order: means, scales, quaternions, opacities, colours, dL/dpixel.  The
five named presets restate the synthetic workloads the rasterizer is measured
on: 256 Gaussians at 64x64 up to 3M Gaussians at 1920x1080 seen by four
cameras.  The pages measure on no public dataset, so none is stood in for.

Scene parameters are the *activated* values the rasterizer consumes: linear
scales (already exp'd), unit-ish quaternions (w, x, y, z), opacities in (0, 1)
(already sigmoid'ed) and RGB colours.  Activation functions belong to the
user's model, not to the rasterizer.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

# Rasterizer constants shared by the presets.  Each is a field of the camera
# record so that the oracle and the CUDA path receive the same value.
DEFAULT_TILE = 16
DEFAULT_Z_NEAR = 0.2
DEFAULT_EPS2D = 0.3          # low-pass dilation added to the 2D covariance (px^2)
DEFAULT_ALPHA_MAX = 0.99     # opacity cap, given on the pages
DEFAULT_ALPHA_MIN = 1.0 / 255.0
DEFAULT_T_MIN = 1e-4
DEFAULT_SIGMA_MULT = 3.0     # support radius in standard deviations


@dataclasses.dataclass
class Camera:
    """Pinhole camera plus the rasterizer's scalar parameters.

    ``R`` (row-major 3x3) and ``t`` map world to camera coordinates:
    x_cam = R @ x_world + t.  Pixel (x, y) has its centre at (x + 0.5, y + 0.5).
    """
    width: int
    height: int
    fx: float
    fy: float
    cx: float
    cy: float
    R: Sequence[float] = (1.0, 0.0, 0.0, 0.0, 1.0, 0.0, 0.0, 0.0, 1.0)
    t: Sequence[float] = (0.0, 0.0, 0.0)
    tile: int = DEFAULT_TILE
    z_near: float = DEFAULT_Z_NEAR
    eps2d: float = DEFAULT_EPS2D
    alpha_max: float = DEFAULT_ALPHA_MAX
    alpha_min: float = DEFAULT_ALPHA_MIN
    T_min: float = DEFAULT_T_MIN
    sigma_mult: float = DEFAULT_SIGMA_MULT
    bg: Sequence[float] = (0.0, 0.0, 0.0)

    @property
    def tiles_x(self) -> int:
        return (self.width + self.tile - 1) // self.tile

    @property
    def tiles_y(self) -> int:
        return (self.height + self.tile - 1) // self.tile

    @property
    def num_tiles(self) -> int:
        return self.tiles_x * self.tiles_y

    def replace(self, **kw) -> "Camera":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass
class Scene:
    """One seeded scene: float32 parameters, one or more cameras and the
    upstream image gradient per camera ([3, H, W], channel-major)."""
    name: str
    means: np.ndarray        # [N, 3] float32
    scales: np.ndarray       # [N, 3] float32, linear
    quats: np.ndarray        # [N, 4] float32, (w, x, y, z)
    opacity: np.ndarray      # [N] float32, in (0, 1)
    colors: np.ndarray       # [N, 3] float32, RGB
    cameras: List[Camera]
    dL_dimage: List[np.ndarray]  # per camera: [3, H, W] float32

    @property
    def N(self) -> int:
        return int(self.means.shape[0])


def _unit_quats(rng: np.random.Generator, n: int) -> np.ndarray:
    q = rng.standard_normal((n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    return q


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def _clustered_means(rng: np.random.Generator, n: int, k: int, sigma: float,
                     lo: Sequence[float], hi: Sequence[float]) -> np.ndarray:
    centres = rng.uniform(lo, hi, size=(k, 3))
    which = rng.integers(0, k, size=n)
    return centres[which] + sigma * rng.standard_normal((n, 3))


def _yaw(deg: float) -> tuple:
    """Row-major rotation about the camera's y axis by ``deg`` degrees."""
    a = math.radians(deg)
    c, s = math.cos(a), math.sin(a)
    return (c, 0.0, s, 0.0, 1.0, 0.0, -s, 0.0, c)


def _finish(name, rng, means, scales, quats, op_std, cams, dl_std) -> Scene:
    n = means.shape[0]
    opacity = _sigmoid(op_std * rng.standard_normal(n))
    colors = rng.uniform(0.0, 1.0, size=(n, 3))
    dls = [(dl_std * rng.standard_normal((3, c.height, c.width))).astype(np.float32)
           for c in cams]
    return Scene(name=name,
                 means=np.ascontiguousarray(means, dtype=np.float32),
                 scales=np.ascontiguousarray(scales, dtype=np.float32),
                 quats=np.ascontiguousarray(quats, dtype=np.float32),
                 opacity=np.ascontiguousarray(opacity, dtype=np.float32),
                 colors=np.ascontiguousarray(colors, dtype=np.float32),
                 cameras=cams, dL_dimage=dls)


def config1(seed: int = 0) -> Scene:
    """256 Gaussians, 64x64, f = 64, identity view; means U([-1,1]^2 x [3,5])."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n = 256
    means = rng.uniform((-1, -1, 3), (1, 1, 5), size=(n, 3))
    scales = np.exp(rng.normal(-3.0, 0.5, size=(n, 3)))
    quats = _unit_quats(rng, n)
    cam = Camera(64, 64, 64.0, 64.0, 32.0, 32.0)
    return _finish("cfg1_256_64x64", rng, means, scales, quats, 1.0, [cam], 1.0)


def config2(seed: int = 0) -> Scene:
    """10k Gaussians, 256x256, f = 256; means U([-2,2]^2 x [3,8])."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n = 10_000
    means = rng.uniform((-2, -2, 3), (2, 2, 8), size=(n, 3))
    scales = np.exp(rng.normal(-3.5, 0.5, size=(n, 3)))
    quats = _unit_quats(rng, n)
    cam = Camera(256, 256, 256.0, 256.0, 128.0, 128.0)
    return _finish("cfg2_10k_256x256", rng, means, scales, quats, 1.0, [cam], 1.0)


def config3(seed: int = 0) -> Scene:
    """100k Gaussians, 800x800, f = 1100; 32 clusters (sigma 0.3) in [-2,2]^2 x [3,10]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n = 100_000
    means = _clustered_means(rng, n, 32, 0.3, (-2, -2, 3), (2, 2, 10))
    scales = np.exp(rng.normal(-4.0, 0.6, size=(n, 3)))
    quats = _unit_quats(rng, n)
    cam = Camera(800, 800, 1100.0, 1100.0, 400.0, 400.0)
    return _finish("cfg3_100k_800x800", rng, means, scales, quats, 1.5, [cam], 0.1)


def config4(seed: int = 0) -> Scene:
    """1M Gaussians, 1920x1080, f = 1600; 256 clusters (sigma 0.2) in [-3,3]x[-2,2]x[2,15]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n = 1_000_000
    means = _clustered_means(rng, n, 256, 0.2, (-3, -2, 2), (3, 2, 15))
    scales = np.exp(rng.normal(-4.5, 0.7, size=(n, 3)))
    quats = _unit_quats(rng, n)
    cam = Camera(1920, 1080, 1600.0, 1600.0, 960.0, 540.0)
    return _finish("cfg4_1M_1920x1080", rng, means, scales, quats, 1.5, [cam], 0.1)


def config5(seed: int = 0, n: int = 3_000_000) -> Scene:
    """3M Gaussians, 1920x1080, four cameras (yaw 0, +10, -10, +20 degrees).

    A seeded subset of exactly floor(0.1 N) Gaussians is large
    (scales exp(N(-1.5, 0.5))); the rest are small (exp(N(-5, 0.7))).  Means
    are 1024 clusters with the 1M scene's sigma and box.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    means = _clustered_means(rng, n, 1024, 0.2, (-3, -2, 2), (3, 2, 15))
    scales = np.exp(rng.normal(-5.0, 0.7, size=(n, 3)))
    big = rng.permutation(n)[: n // 10]
    scales[big] = np.exp(rng.normal(-1.5, 0.5, size=(big.size, 3)))
    quats = _unit_quats(rng, n)
    cams = [Camera(1920, 1080, 1600.0, 1600.0, 960.0, 540.0, R=_yaw(d))
            for d in (0.0, 10.0, -10.0, 20.0)]
    return _finish(f"cfg5_{n // 1000}k_1920x1080_x4", rng, means, scales, quats, 2.0, cams, 0.1)


PRESETS = {1: config1, 2: config2, 3: config3, 4: config4, 5: config5}


def preset(index: int, seed: int = 0) -> Scene:
    return PRESETS[index](seed)


def random_tiny(n: int = 6, width: int = 32, height: int = 32, seed: int = 0,
                opacity_max: float = 0.9, scale_log_mean: float = -2.0,
                z_range=(2.5, 4.5), sigma_mult: float = 3.0,
                alpha_min: float = DEFAULT_ALPHA_MIN, T_min: float = DEFAULT_T_MIN,
                distinct_depth_gap: Optional[float] = 0.05) -> Scene:
    """A tiny scene for finite-difference and brute-force checks.

    Depths are spread so that no two are closer than ``distinct_depth_gap``
    (sort order then cannot flip under a 1e-4 perturbation), and opacities stay
    below ``opacity_max`` so that the 0.99 cap is never reached.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    f = float(width)
    means = np.empty((n, 3))
    means[:, 0] = rng.uniform(-0.5, 0.5, n)
    means[:, 1] = rng.uniform(-0.5, 0.5, n)
    if distinct_depth_gap is None:
        means[:, 2] = rng.uniform(z_range[0], z_range[1], n)
    else:
        base = np.linspace(z_range[0], z_range[1], n)
        means[:, 2] = rng.permutation(base)
    scales = np.exp(rng.normal(scale_log_mean, 0.4, size=(n, 3)))
    quats = _unit_quats(rng, n)
    opacity = rng.uniform(0.2, opacity_max, n)
    colors = rng.uniform(0.0, 1.0, size=(n, 3))
    cam = Camera(width, height, f, f, width / 2.0, height / 2.0,
                 sigma_mult=sigma_mult, alpha_min=alpha_min, T_min=T_min)
    dl = rng.standard_normal((3, height, width))
    return Scene(name=f"tiny_{n}_{width}x{height}_s{seed}",
                 means=means.astype(np.float32), scales=scales.astype(np.float32),
                 quats=quats.astype(np.float32), opacity=opacity.astype(np.float32),
                 colors=colors.astype(np.float32), cameras=[cam],
                 dL_dimage=[dl.astype(np.float32)])


def random_sh(n: int, degree: int, seed: int = 0, dc_max: float = 3.0, rest_std: float = 0.2) -> np.ndarray:
    """Seeded spherical-harmonics coefficients [n, (degree+1)^2, 3] (float32):
    the constant band uniform in [0, dc_max), the others normal(0, rest_std)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    K = (degree + 1) ** 2
    sh = rng.normal(0.0, rest_std, size=(n, K, 3))
    sh[:, 0, :] = rng.uniform(0.0, dc_max, size=(n, 3))
    return np.ascontiguousarray(sh, dtype=np.float32)
