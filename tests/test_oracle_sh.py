"""Pins of the oracle's spherical-harmonics colour (the colour -> SH step of
the page 'Gaussian Splatting反向传播的CUDA实现', section 4) to mathematics."""
import math

import numpy as np
import pytest

import oracle
from differentiable_gaussian_splatting_preprocess_b200 import scenes


def _sphere_quadrature(nz=8, nphi=16):
    """Gauss-Legendre in z times uniform in phi: exact for polynomials of
    degree < 2 nz in z and < nphi in the azimuthal frequency."""
    z, wz = np.polynomial.legendre.leggauss(nz)
    phi = np.arange(nphi) * 2 * np.pi / nphi
    Z, PHI = np.meshgrid(z, phi, indexing="ij")
    r = np.sqrt(1 - Z ** 2)
    d = np.stack([r * np.cos(PHI), r * np.sin(PHI), Z], -1).reshape(-1, 3)
    w = (wz[:, None] * np.full(nphi, 2 * np.pi / nphi)[None, :]).reshape(-1)
    return d, w


def test_basis_is_orthonormal_on_the_sphere():
    d, w = _sphere_quadrature()
    Y = oracle.sh_basis(d)
    gram = (Y * w[:, None]).T @ Y
    np.testing.assert_allclose(gram, np.eye(16), atol=1e-12)


def test_addition_theorem_per_band():
    """sum_m Y_lm(d)^2 = (2l + 1) / (4 pi) for every unit direction."""
    rng = np.random.default_rng(0)
    d = rng.normal(size=(100, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    Y = oracle.sh_basis(d)
    for l in range(4):
        band = Y[:, l * l:(l + 1) * (l + 1)]
        np.testing.assert_allclose((band ** 2).sum(1), (2 * l + 1) / (4 * math.pi), rtol=1e-12)


def test_degree0_and_degree1_closed_forms():
    cam = scenes.Camera(32, 32, 32.0, 32.0, 16.0, 16.0, t=(0.0, 0.0, 0.0))
    mean = np.array([[0.3, -0.4, 1.2]])
    d = mean[0] / np.linalg.norm(mean[0])
    sh = np.zeros((1, 4, 3))
    sh[0, 0] = [1.0, 2.0, 0.5]
    sh[0, 1:] = [[0.1, 0.0, 0.3], [0.2, -0.1, 0.0], [-0.3, 0.2, 0.1]]
    c0 = 1 / (2 * math.sqrt(math.pi))
    c1 = math.sqrt(3 / (4 * math.pi))
    got0 = oracle.sh_fwd(cam, mean, sh[:, :1], 0, offset=0.5)
    np.testing.assert_allclose(got0[0], c0 * sh[0, 0] + 0.5, rtol=1e-14)
    got1 = oracle.sh_fwd(cam, mean, sh, 1, offset=0.5)
    want = c0 * sh[0, 0] + c1 * (d[1] * sh[0, 1] + d[2] * sh[0, 2] + d[0] * sh[0, 3]) + 0.5
    np.testing.assert_allclose(got1[0], want, rtol=1e-13)


def test_colour_depends_on_direction_only():
    """Moving the camera centre and the means together leaves colours unchanged;
    scaling the distance along the ray does too."""
    rng = np.random.default_rng(1)
    sh = scenes.random_sh(20, 3, seed=2).astype(np.float64)
    means = rng.normal(size=(20, 3)) + [0, 0, 4]
    cam = scenes.Camera(32, 32, 32.0, 32.0, 16.0, 16.0)
    a = oracle.sh_fwd(cam, means, sh, 3, 0.5)
    shift = np.array([0.25, -0.5, 0.125])
    cam2 = cam.replace(t=tuple(-shift))  # identity R: camera centre = -t = shift
    b = oracle.sh_fwd(cam2, means + shift, sh, 3, 0.5)
    c = oracle.sh_fwd(cam, means * 1.75, sh, 3, 0.5)
    np.testing.assert_allclose(b, a, atol=1e-12)
    np.testing.assert_allclose(c, a, atol=1e-12)


@pytest.mark.parametrize("degree", [0, 1, 2, 3])
def test_sh_gradients_match_central_differences(degree):
    rng = np.random.default_rng(degree)
    n = 5
    cam = scenes.Camera(32, 32, 32.0, 32.0, 16.0, 16.0, R=(0.96, 0.0, 0.28, 0.0, 1.0, 0.0, -0.28, 0.0, 0.96),
                        t=(0.1, -0.2, 0.3))
    means = rng.normal(size=(n, 3)) + [0, 0, 3]
    sh = scenes.random_sh(n, degree, seed=degree + 10).astype(np.float64)
    sh[0, 0, 1] = -5.0  # one clamped channel: its gradient must vanish
    g = rng.normal(size=(n, 3))
    loss = lambda m, s: float((oracle.sh_fwd(cam, m, s, degree, 0.5) * g).sum())
    an = oracle.sh_bwd(cam, means, sh, degree, g, 0.5)
    eps = 1e-4
    for name, x in (("dL_dmeans", means), ("dL_dsh", sh)):
        fd = np.zeros_like(x)
        for i in range(x.size):
            xp, xm = x.copy(), x.copy()
            xp.reshape(-1)[i] += eps
            xm.reshape(-1)[i] -= eps
            args_p = (xp, sh) if name == "dL_dmeans" else (means, xp)
            args_m = (xm, sh) if name == "dL_dmeans" else (means, xm)
            fd.reshape(-1)[i] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(an[name], fd, atol=1e-6 * max(1.0, np.abs(fd).max()), err_msg=name)
    assert not an["dL_dsh"][0, :, 1].any()


def test_full_pipeline_gradient_through_sh_colours():
    """Render with colours from SH: the gradient w.r.t. means gathers the
    geometric path and the view-direction path; both checked against central
    differences of the whole forward."""
    sc = scenes.random_tiny(n=5, seed=8, sigma_mult=50.0, alpha_min=0.0, T_min=0.0)
    cam = sc.cameras[0]
    sh = scenes.random_sh(sc.N, 2, seed=3).astype(np.float64)
    g = sc.dL_dimage[0].astype(np.float64)
    P = dict(means=sc.means.astype(np.float64), sh=sh)

    def loss(Q):
        col = oracle.sh_fwd(cam, Q["means"], Q["sh"], 2, 0.5)
        f = oracle.forward(cam, Q["means"], sc.scales, sc.quats, sc.opacity, col, "f64")
        return float((f["image"] * g).sum())

    col = oracle.sh_fwd(cam, P["means"], sh, 2, 0.5)
    fb = oracle.forward_backward(cam, P["means"], sc.scales, sc.quats, sc.opacity, col, g, "f64")
    shb = oracle.sh_bwd(cam, P["means"], sh, 2, fb["dL_dcolors"], 0.5)
    an = dict(means=fb["dL_dmeans"] + shb["dL_dmeans"], sh=shb["dL_dsh"])
    eps = 1e-4
    for k in ("means", "sh"):
        fd = np.zeros_like(P[k])
        for i in range(P[k].size):
            Qp = {kk: v.copy() for kk, v in P.items()}
            Qm = {kk: v.copy() for kk, v in P.items()}
            Qp[k].reshape(-1)[i] += eps
            Qm[k].reshape(-1)[i] -= eps
            fd.reshape(-1)[i] = (loss(Qp) - loss(Qm)) / (2 * eps)
        np.testing.assert_allclose(an[k], fd, atol=1e-5 * np.abs(fd).max(), err_msg=k)
