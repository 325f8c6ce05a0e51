"""Parity of the spherical-harmonics colour kernels (gs_sh_fwd / gs_sh_bwd)
with the oracle, alone and inside the whole forward + backward."""
import numpy as np
import pytest
import torch

import oracle
from differentiable_gaussian_splatting_preprocess_b200 import binding as B
from differentiable_gaussian_splatting_preprocess_b200 import rasterizer as RZ
from differentiable_gaussian_splatting_preprocess_b200 import scenes

from _gpu_pipeline import GRAD_REL_L2, GpuScene, rel_l2, to_dev, to_np

pytestmark = pytest.mark.gpu


def _rotated_cam(cam):
    return cam.replace(R=(0.96, 0.0, 0.28, 0.0, 1.0, 0.0, -0.28, 0.0, 0.96), t=(0.1, -0.2, 0.3))


@pytest.mark.parametrize("degree", [0, 1, 2, 3])
def test_sh_colours_and_gradients(degree):
    sc = scenes.preset(3)
    cam = _rotated_cam(sc.cameras[0])
    K = 16  # stored coefficients; only (degree + 1)^2 are read
    sh = scenes.random_sh(sc.N, 3, seed=degree)
    sh[:50, 0, :] = -5.0  # clamped colours
    means, shd = to_dev(sc.means), to_dev(sh)
    col = torch.empty((sc.N, 3), device="cuda")
    B.gs_sh_fwd(cam, degree, means, shd, col, offset=0.5)
    g = np.random.default_rng(degree).normal(size=(sc.N, 3)).astype(np.float32)
    dsh = torch.zeros_like(shd)
    dmu = torch.zeros_like(means)
    B.gs_sh_bwd(cam, degree, means, shd, to_dev(g), dsh, dmu, offset=0.5)
    torch.cuda.synchronize()
    o32 = oracle.sh_fwd(cam, sc.means, sh, degree, 0.5, "f32")
    o64 = oracle.sh_fwd(cam, sc.means, sh, degree, 0.5, "f64")
    np.testing.assert_allclose(to_np(col), o32, atol=5e-6)
    np.testing.assert_allclose(to_np(col), o64, atol=1e-5)
    assert not to_np(col)[:50].any()
    ob = oracle.sh_bwd(cam, sc.means, sh, degree, g, 0.5, "f64")
    assert rel_l2(to_np(dsh), ob["dL_dsh"]) <= 1e-5
    assert rel_l2(to_np(dmu), ob["dL_dmeans"]) <= 1e-4
    assert not to_np(dsh)[:, (degree + 1) ** 2:].any()
    assert not to_np(dsh)[:50].any()


@pytest.mark.parametrize("cfg", [2, 3])
def test_render_with_sh_colours_end_to_end(cfg):
    sc = scenes.preset(cfg)
    cam = _rotated_cam(sc.cameras[0])
    degree = 3
    sh = scenes.random_sh(sc.N, degree, seed=7)
    gs = GpuScene(sc)
    shd = to_dev(sh)
    col = torch.empty((sc.N, 3), device="cuda")
    B.gs_sh_fwd(cam, degree, gs.means, shd, col, offset=0.5)
    rz = RZ.Rasterizer(cam)
    fr = rz.forward(gs.means, gs.scales, gs.quats, gs.opacity, col)
    g = rz.backward(fr, gs.means, gs.scales, gs.quats, col, to_dev(sc.dL_dimage[0]))
    dsh = torch.zeros_like(shd)
    B.gs_sh_bwd(cam, degree, gs.means, shd, g["dL_dcolors"], dsh, g["dL_dmeans"], offset=0.5)
    torch.cuda.synchronize()
    ocol = oracle.sh_fwd(cam, sc.means, sh, degree, 0.5, "f64")
    f = oracle.forward_backward(cam, sc.means, sc.scales, sc.quats, sc.opacity, ocol, sc.dL_dimage[0], "f64")
    ob = oracle.sh_bwd(cam, sc.means, sh, degree, f["dL_dcolors"], 0.5, "f64")
    assert rel_l2(to_np(g["dL_dmeans"]), f["dL_dmeans"] + ob["dL_dmeans"]) <= GRAD_REL_L2
    assert rel_l2(to_np(dsh), ob["dL_dsh"]) <= GRAD_REL_L2
    for k in ("dL_dscales", "dL_dquats", "dL_dopacity"):
        assert rel_l2(to_np(g[k]), f[k]) <= GRAD_REL_L2, k


@pytest.mark.parametrize("degree", [1, 3])
def test_sh_half_precision_storage(degree):
    """gs_sh_*_f16: coefficients stored as binary16, arithmetic in fp32.  The
    bar is the fp32 one, against the oracle evaluated on the widened
    coefficients (binary16 -> float64 is exact); the distance to the
    full-precision colours is the storage rounding alone, at most
    sum_k |Y_k| |sh_k| 2^-11 per channel."""
    sc = scenes.preset(3)
    cam = _rotated_cam(sc.cameras[0])
    sh = scenes.random_sh(sc.N, degree, seed=11 + degree)
    sh[:40, 0, :] = -5.0
    sh16 = sh.astype(np.float16)
    wide = sh16.astype(np.float64)
    means = to_dev(sc.means)
    shd16 = torch.from_numpy(sh16).cuda()
    col = torch.empty((sc.N, 3), device="cuda")
    B.gs_sh_fwd(cam, degree, means, shd16, col, offset=0.5)
    g = np.random.default_rng(degree).normal(size=(sc.N, 3)).astype(np.float32)
    dsh = torch.zeros(sh.shape, dtype=torch.float32, device="cuda")
    dmu = torch.zeros_like(means)
    B.gs_sh_bwd_f16(cam, degree, means, shd16, to_dev(g), dsh, dmu, offset=0.5)
    torch.cuda.synchronize()
    o64 = oracle.sh_fwd(cam, sc.means, wide, degree, 0.5, "f64")
    np.testing.assert_allclose(to_np(col), o64, atol=1e-5)
    assert not to_np(col)[:40].any()
    ob = oracle.sh_bwd(cam, sc.means, wide, degree, g, 0.5, "f64")
    assert rel_l2(to_np(dsh), ob["dL_dsh"]) <= 1e-5
    assert rel_l2(to_np(dmu), ob["dL_dmeans"]) <= 1e-4
    # storage rounding relative to the full-precision coefficients
    full = oracle.sh_fwd(cam, sc.means, sh.astype(np.float64), degree, 0.5, "f64")
    R = np.asarray(cam.R, np.float64).reshape(3, 3)
    v = sc.means.astype(np.float64) + R.T @ np.asarray(cam.t, np.float64)  # mean - camera centre
    Y = np.abs(oracle.sh_basis(v / np.linalg.norm(v, axis=1, keepdims=True)))[:, :(degree + 1) ** 2]
    bound = np.einsum("nk,nkc->nc", Y, np.abs(sh[:, :(degree + 1) ** 2].astype(np.float64))) * 2.0 ** -11
    assert np.all(np.abs(to_np(col) - full) <= bound + 1e-5)
    with pytest.raises(TypeError):
        B.gs_sh_fwd_f16(cam, degree, means, to_dev(sh), col)
