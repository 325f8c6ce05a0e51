"""Pins of the CPU oracle to the pages and to mathematics (no GPU).

Each test checks the oracle against something other than itself: closed forms,
hand-derived golden values, brute force with no tiling, invariants and float64
central differences with eps = 1e-4 (the gradient check recommended on the page
'Gaussian Splatting反向传播的CUDA实现', section 6).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from differentiable_gaussian_splatting_preprocess_b200 import scenes

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32(x):
    """Camera parameters travel as float32; closed forms use the same value."""
    return float(np.float32(x))


def _cam(w=32, h=32, f=32.0, **kw):
    return scenes.Camera(w, h, f, f, w / 2.0, h / 2.0, **kw)


def _iso(n, s=0.1):
    return np.full((n, 3), s, np.float64)


def _ident_q(n):
    q = np.zeros((n, 4))
    q[:, 0] = 1.0
    return q


def _rot_from_quat(q):
    """Rotation of a unit quaternion by Rodrigues' formula (axis-angle), a route
    independent of the quaternion-product matrix the oracle uses."""
    q = np.asarray(q, np.float64)
    q = q / np.linalg.norm(q)
    w, v = q[0], q[1:]
    s = np.linalg.norm(v)
    if s == 0:
        return np.eye(3)
    axis = v / s
    ang = 2.0 * math.atan2(s, w)
    K = np.array([[0, -axis[2], axis[1]], [axis[2], 0, -axis[0]], [-axis[1], axis[0], 0]])
    return np.eye(3) + math.sin(ang) * K + (1 - math.cos(ang)) * (K @ K)


# --------------------------------------------------------------------------
# Preprocess: projection, covariance, conic, radius, rectangle
# --------------------------------------------------------------------------

@pytest.mark.parametrize("mode", ["f32", "f64"])
def test_on_axis_covariance_closed_form(mode):
    """Mean on the optical axis, identity view and rotation: Sigma2 is
    diag(fx^2 sx^2 / z^2, fy^2 sy^2 / z^2) + eps I, so the conic is its inverse."""
    cam = scenes.Camera(64, 48, 40.0, 50.0, 32.0, 24.0)
    z, sx, sy, sz = 3.0, 0.05, 0.08, 0.2
    pre = oracle.preprocess(cam, [[0, 0, z]], [[sx, sy, sz]], [[1, 0, 0, 0]], [0.7], mode)
    a = (40.0 * sx / z) ** 2 + _f32(cam.eps2d)
    c = (50.0 * sy / z) ** 2 + _f32(cam.eps2d)
    tol = 1e-6 if mode == "f32" else 1e-12
    np.testing.assert_allclose(pre["conic_opacity"][0], [1 / a, 0.0, 1 / c, 0.7], rtol=tol, atol=tol)
    np.testing.assert_allclose(pre["mean2d"][0], [32.0, 24.0], rtol=0, atol=0)
    assert pre["depth"][0] == pytest.approx(z)
    r = math.ceil(3 * math.sqrt(max(a, c)))
    assert pre["radius"][0] == r
    # rectangle [floor((u - r)/16), ceil((u + r)/16)) clamped to the tile grid
    x0, x1 = max(0, math.floor((32 - r) / 16)), min(4, math.ceil((32 + r) / 16))
    y0, y1 = max(0, math.floor((24 - r) / 16)), min(3, math.ceil((24 + r) / 16))
    assert list(pre["rect"][0]) == [x0, y0, x1, y1]
    assert pre["tiles_touched"][0] == (x1 - x0) * (y1 - y0)


@pytest.mark.parametrize("mode", ["f32", "f64"])
def test_quaternion_90deg_about_z_swaps_axes(mode):
    """R(q) for 90 degrees about z maps x to y, so anisotropic scales swap in
    the projected covariance."""
    cam = scenes.Camera(64, 64, 40.0, 40.0, 32.0, 32.0)
    z, sx, sy = 4.0, 0.05, 0.15
    h = math.sqrt(0.5)
    pre = oracle.preprocess(cam, [[0, 0, z]], [[sx, sy, 0.1]], [[h, 0, 0, h]], [0.5], mode)
    a = (40.0 * sy / z) ** 2 + _f32(cam.eps2d)
    c = (40.0 * sx / z) ** 2 + _f32(cam.eps2d)
    tol = 1e-5 if mode == "f32" else 1e-12
    np.testing.assert_allclose(pre["conic_opacity"][0, [0, 2]], [1 / a, 1 / c], rtol=tol)
    assert abs(pre["conic_opacity"][0, 1]) < tol * 10


def test_off_axis_isotropic_closed_form():
    """Mean at (x, 0, z), isotropic scale s: Sigma2 = s^2 J J^T + eps I with the
    pinhole Jacobian J = [[f/z, 0, -f x/z^2], [0, f/z, 0]]; u = f x / z + cx."""
    f, x, z, s = 30.0, 0.7, 2.5, 0.06
    cam = scenes.Camera(64, 64, f, f, 32.0, 32.0)
    pre = oracle.preprocess(cam, [[x, 0, z]], [[s, s, s]], [[0.3, 0.5, -0.2, 0.7]], [0.5], "f64")
    S2 = s * s * np.array([[f * f / z ** 2 + (f * x / z ** 2) ** 2, 0.0], [0.0, f * f / z ** 2]]) + _f32(cam.eps2d) * np.eye(2)
    A = np.linalg.inv(S2)
    np.testing.assert_allclose(pre["conic_opacity"][0, :3], [A[0, 0], A[0, 1], A[1, 1]], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(pre["mean2d"][0], [f * x / z + 32.0, 32.0], rtol=1e-14)


def test_general_covariance_matches_rodrigues():
    """Random scene, rotated camera: the oracle's conic equals the inverse of
    J W R S S^T R^T W^T J^T + eps I built with numpy from an axis-angle
    rotation (Rodrigues) instead of the quaternion-product matrix."""
    rng = np.random.default_rng(5)
    cam = scenes.Camera(96, 80, 70.0, 60.0, 45.0, 41.0)
    Wc = _rot_from_quat([0.95, 0.1, -0.2, 0.15])
    cam = cam.replace(R=tuple(Wc.reshape(-1)), t=(0.2, -0.1, 0.5))
    Wc = np.asarray(cam.R, np.float32).astype(np.float64).reshape(3, 3)   # as the camera record holds it
    tc = np.asarray(cam.t, np.float32).astype(np.float64)
    n = 20
    means = np.c_[rng.uniform(-0.5, 0.5, (n, 2)), rng.uniform(2, 4, n)]
    scales = np.exp(rng.normal(-2.5, 0.4, (n, 3)))
    quats = rng.normal(size=(n, 4)) * 2.3
    pre = oracle.preprocess(cam, means, scales, quats, np.full(n, 0.5), "f64")
    for i in range(n):
        t = Wc @ means[i] + tc
        J = np.array([[cam.fx / t[2], 0, -cam.fx * t[0] / t[2] ** 2], [0, cam.fy / t[2], -cam.fy * t[1] / t[2] ** 2]])
        R = _rot_from_quat(quats[i])
        S3 = R @ np.diag(scales[i] ** 2) @ R.T
        S2 = J @ Wc @ S3 @ Wc.T @ J.T + _f32(cam.eps2d) * np.eye(2)
        A = np.linalg.inv(S2)
        if pre["radius"][i] == 0:
            continue
        np.testing.assert_allclose(pre["conic_opacity"][i, :3], [A[0, 0], A[0, 1], A[1, 1]], rtol=1e-10)
        np.testing.assert_allclose(pre["mean2d"][i], [cam.fx * t[0] / t[2] + cam.cx, cam.fy * t[1] / t[2] + cam.cy],
                                   rtol=1e-12)
        lam = np.linalg.eigvalsh(S2).max()
        assert pre["radius"][i] == math.ceil(3 * math.sqrt(lam))


def test_isotropic_covariance_independent_of_rotation():
    """R R^T = I: with isotropic scales the conic does not depend on q."""
    rng = np.random.default_rng(1)
    cam = _cam(64, 64, 50.0)
    n = 16
    means = np.tile([[0.1, -0.05, 3.0]], (n, 1))
    scales = _iso(n, 0.07)
    quats = rng.normal(size=(n, 4))
    pre = oracle.preprocess(cam, means, scales, quats, np.full(n, 0.5), "f64")
    np.testing.assert_allclose(pre["conic_opacity"], np.tile(pre["conic_opacity"][:1], (n, 1)), rtol=1e-12)


def test_camera_transform_equivalence():
    """A camera (W, t) seeing mu equals the identity camera seeing W mu + t
    when the Gaussian is isotropic."""
    Wc = _rot_from_quat([0.9, -0.1, 0.3, 0.2]).astype(np.float32).astype(np.float64)
    t = np.array([0.3, -0.2, 0.4], np.float32).astype(np.float64)
    cam = _cam(64, 64, 50.0).replace(R=tuple(Wc.reshape(-1)), t=tuple(t))
    cam0 = _cam(64, 64, 50.0)
    mu = np.array([[0.2, 0.1, 2.5]])
    pre = oracle.preprocess(cam, mu, _iso(1, 0.05), _ident_q(1), [0.5], "f64")
    pre0 = oracle.preprocess(cam0, (Wc @ mu[0] + t)[None], _iso(1, 0.05), _ident_q(1), [0.5], "f64")
    for k in ("mean2d", "depth", "conic_opacity"):
        np.testing.assert_allclose(pre[k], pre0[k], rtol=1e-12)


@pytest.mark.parametrize("mode", ["f32", "f64"])
def test_culling_rules(mode):
    cam = _cam(32, 32, 32.0)
    means = [[0, 0, 0.1],      # in front of the camera but nearer than z_near
             [0, 0, -3.0],     # behind
             [100, 0, 3.0],    # far outside the image
             [0, 0, 3.0],      # zero quaternion
             [0, 0, 3.0]]      # visible
    quats = [[1, 0, 0, 0]] * 3 + [[0, 0, 0, 0], [1, 0, 0, 0]]
    pre = oracle.preprocess(cam, means, _iso(5, 0.05), quats, [0.5] * 5, mode)
    assert list(pre["radius"][:4]) == [0, 0, 0, 0]
    assert list(pre["tiles_touched"][:4]) == [0, 0, 0, 0]
    assert not pre["conic_opacity"][:4].any() and not pre["mean2d"][:4].any()
    assert pre["radius"][4] > 0 and pre["tiles_touched"][4] > 0


# --------------------------------------------------------------------------
# Binning
# --------------------------------------------------------------------------

def _brute_lists(cam, pre):
    """For every tile, the Gaussians whose rectangle contains it, ordered by
    (depth, id) with numpy's lexsort."""
    TX, TY = cam.tiles_x, cam.tiles_y
    rect, depth, tt = pre["rect"], pre["depth"], pre["tiles_touched"]
    out = []
    for t in range(TX * TY):
        tx, ty = t % TX, t // TX
        m = (tt > 0) & (rect[:, 0] <= tx) & (tx < rect[:, 2]) & (rect[:, 1] <= ty) & (ty < rect[:, 3])
        idx = np.nonzero(m)[0]
        order = np.lexsort((idx, depth[idx]))
        out.append(idx[order].astype(np.uint32))
    return out


@pytest.mark.parametrize("cfg", [1, 2])
def test_binning_against_brute_force(cfg):
    sc = scenes.preset(cfg)
    cam = sc.cameras[0]
    pre = oracle.preprocess(cam, sc.means, sc.scales, sc.quats, sc.opacity, "f32")
    b = oracle.bin_pairs(cam, pre["depth"], pre["rect"], pre["tiles_touched"], "f32")
    keys, ids, ranges = b["keys"], b["ids"], b["ranges"]
    assert b["num_pairs"] == int(pre["tiles_touched"].sum())
    assert np.all(keys[1:] >= keys[:-1])
    # ranges partition [0, P) in tile order; empty tiles are (0, 0)
    pos = 0
    for t in range(cam.num_tiles):
        s, e = ranges[t]
        if s == e:
            assert s == 0 and e == 0
            continue
        assert s == pos
        pos = e
    assert pos == b["num_pairs"]
    brute = _brute_lists(cam, pre)
    for t in range(cam.num_tiles):
        s, e = ranges[t]
        np.testing.assert_array_equal(ids[s:e], brute[t])
        assert np.all((keys[s:e] >> np.uint64(32)) == t)
        np.testing.assert_array_equal((keys[s:e] & np.uint64(0xFFFFFFFF)).astype(np.uint32),
                                      pre["depth"][ids[s:e]].view(np.uint32))
    for t in (0, cam.num_tiles // 2, cam.num_tiles - 1):
        np.testing.assert_array_equal(oracle.tile_list(cam, pre["depth"], pre["rect"], pre["tiles_touched"], t),
                                      brute[t])


def test_equal_depth_ties_broken_by_id():
    cam = _cam(32, 32, 32.0)
    n = 5
    means = np.tile([[0.0, 0.0, 3.0]], (n, 1))
    pre = oracle.preprocess(cam, means, _iso(n, 0.05), _ident_q(n), [0.5] * n, "f32")
    b = oracle.bin_pairs(cam, pre["depth"], pre["rect"], pre["tiles_touched"], "f32")
    for t in range(cam.num_tiles):
        s, e = b["ranges"][t]
        if e > s:
            np.testing.assert_array_equal(b["ids"][s:e], np.arange(n))


# --------------------------------------------------------------------------
# Compositing forward
# --------------------------------------------------------------------------

@pytest.mark.parametrize("mode", ["f32", "f64"])
def test_golden_compositing(mode):
    with open(os.path.join(GOLDEN, "compositing_cases.json")) as fh:
        g = json.load(fh)
    c = g["camera"]
    px, py = g["pixel"]
    for case in g["cases"]:
        cam = scenes.Camera(c["width"], c["height"], c["fx"], c["fy"], c["cx"], c["cy"],
                            T_min=case["T_min"], bg=tuple(case["bg"]))
        gs = case["gaussians"]
        n = len(gs)
        f = oracle.forward(cam, np.reshape([x["mean"] for x in gs], (n, 3)), _iso(n, 0.1), _ident_q(n),
                           np.reshape([x["opacity"] for x in gs], (n,)), np.reshape([x["color"] for x in gs], (n, 3)),
                           mode)
        exp = case["expected"]
        tol = max(case["tol"], 1e-7 if mode == "f32" else 1e-12)
        np.testing.assert_allclose(f["image"][:, py, px], exp["color"], atol=tol, err_msg=case["name"])
        assert f["final_T"][py, px] == pytest.approx(exp["final_T"], abs=tol), case["name"]
        assert f["n_contrib"][py, px] == exp["n_contrib"], case["name"]
        assert f["n_blended"][py, px] == exp["n_blended"], case["name"]
        assert f["n_eval"][py, px] == exp["n_eval"], case["name"]


def test_single_gaussian_closed_form():
    """One isotropic Gaussian on the axis: C(p) = c alpha(p) + (1 - alpha(p)) bg
    with alpha = min(0.99, sigma exp(-|d|^2 / (2 s2^2))), s2^2 = f^2 s^2 / z^2 + eps."""
    f, z, s, sig = 32.0, 3.0, 0.2, 0.8
    cam = _cam(32, 32, f, sigma_mult=50.0, alpha_min=0.0, T_min=0.0, bg=(0.1, 0.2, 0.3))
    col = [0.9, 0.4, 0.6]
    out = oracle.forward(cam, [[0, 0, z]], [[s, s, s]], _ident_q(1), [sig], [col], "f64")
    s2 = (f * s / z) ** 2 + _f32(cam.eps2d)
    ys, xs = np.mgrid[0:32, 0:32]
    d2 = (xs + 0.5 - 16.0) ** 2 + (ys + 0.5 - 16.0) ** 2
    alpha = np.minimum(0.99, sig * np.exp(-d2 / (2 * s2)))
    for ch in range(3):
        np.testing.assert_allclose(out["image"][ch], col[ch] * alpha + (1 - alpha) * cam.bg[ch], atol=1e-12)
    np.testing.assert_allclose(out["final_T"], 1 - alpha, atol=1e-12)


@pytest.mark.parametrize("mode,tol", [("f32", 2e-6), ("f64", 1e-12)])
def test_partition_of_unity(mode, tol):
    """Colours = 1 and background = 1: sum_k alpha_k T_k + T_final = 1."""
    sc = scenes.preset(2)
    cam = sc.cameras[0].replace(bg=(1.0, 1.0, 1.0))
    f = oracle.forward(cam, sc.means, sc.scales, sc.quats, sc.opacity, np.ones_like(sc.colors), mode)
    np.testing.assert_allclose(f["image"], 1.0, atol=tol)


@pytest.mark.parametrize("T_min", [1e-4, 0.5])
def test_brute_force_compositing_equals_tiled(T_min):
    """With a support radius large enough that every rectangle covers the
    image, the tiled renderer equals compositing every Gaussian at every pixel
    in (depth, id) order, with no tiles and no binning; so do its work counts
    (entries evaluated, the stopping one included; terms blended) and its
    per-quadrant blend mask.  T_min = 0.5 makes pixels stop early."""
    sc = scenes.random_tiny(n=12, width=48, height=40, seed=7, sigma_mult=1e3, T_min=T_min)
    cam = sc.cameras[0]
    f = oracle.forward(cam, sc.means, sc.scales, sc.quats, sc.opacity, sc.colors, "f64")
    pre = f["pre"]
    assert np.all(pre["tiles_touched"] == cam.num_tiles)
    order = np.lexsort((np.arange(sc.N), pre["depth"]))
    H, W = cam.height, cam.width
    img = np.zeros((3, H, W))
    n_eval = np.zeros((H, W), np.int64)
    n_blend = np.zeros((H, W), np.int64)
    # every tile's list is the whole depth order, so tile t holds list
    # positions t*N .. t*N + N - 1; mask bit of position k in 8x8 quadrant q
    # of its tile: word (k // 32) * 4 + q, bit k % 32
    words = 4 * ((cam.num_tiles * sc.N + 31) // 32)
    mask = np.zeros(words, np.uint32)
    for y in range(H):
        for x in range(W):
            tile = (y // 16) * cam.tiles_x + x // 16
            quad = ((y % 16) // 8) * 2 + (x % 16) // 8
            T, C, last = 1.0, np.zeros(3), 0
            for k, j in enumerate(order):
                n_eval[y, x] += 1
                d = np.array([x + 0.5, y + 0.5]) - pre["mean2d"][j]
                a, b, c, o = pre["conic_opacity"][j]
                power = -0.5 * (a * d[0] ** 2 + c * d[1] ** 2) - b * d[0] * d[1]
                if power > 0:
                    continue
                al = min(cam.alpha_max, o * math.exp(power))
                if al < cam.alpha_min:
                    continue
                if T * (1 - al) < cam.T_min:
                    break
                C += sc.colors[j] * al * T
                T *= 1 - al
                last = k + 1
                n_blend[y, x] += 1
                pos = tile * sc.N + k
                mask[(pos // 32) * 4 + quad] |= np.uint32(1 << (pos % 32))
            img[:, y, x] = C + T * np.array(cam.bg)
            assert f["n_contrib"][y, x] == last
    np.testing.assert_allclose(f["image"], img, atol=1e-12)
    # the work counts and the per-quadrant blend mask, from the same walk
    np.testing.assert_array_equal(f["n_eval"], n_eval)
    np.testing.assert_array_equal(f["n_blended"], n_blend)
    assert (n_eval > n_blend).any()  # alpha_min skips occur
    if T_min > 0.1:
        assert (n_eval < sc.N).any()  # so do stops
    b = f["bins"]
    r = oracle.render_fwd(cam, b["ranges"], b["ids"], pre["mean2d"], pre["conic_opacity"], sc.colors, "f64",
                          blend_mask=True)
    np.testing.assert_array_equal(r["blend_mask"], mask)
    assert mask.any()


def test_translation_by_one_tile():
    """Shifting the principal point by 16 px shifts the image by one tile."""
    sc = scenes.random_tiny(n=10, width=64, height=48, seed=2)
    cam = sc.cameras[0]
    a = oracle.forward(cam, sc.means, sc.scales, sc.quats, sc.opacity, sc.colors, "f64")
    b = oracle.forward(cam.replace(cx=cam.cx + 16.0), sc.means, sc.scales, sc.quats, sc.opacity, sc.colors, "f64")
    np.testing.assert_allclose(b["image"][:, :, 16:], a["image"][:, :, :-16], atol=1e-9)


# --------------------------------------------------------------------------
# Gradients
# --------------------------------------------------------------------------

def _fd_scene(seed, rotated):
    sc = scenes.random_tiny(n=6, seed=seed, sigma_mult=50.0, alpha_min=0.0, T_min=0.0)
    cam = sc.cameras[0]
    if rotated:
        Wc = _rot_from_quat([0.97, 0.05, -0.12, 0.1])
        cam = cam.replace(R=tuple(Wc.reshape(-1)), t=(0.1, -0.05, 0.3), fx=30.0, fy=34.0, cx=15.0, cy=17.5,
                          bg=(0.2, 0.5, 0.9))
    P = dict(means=sc.means.astype(np.float64), scales=sc.scales.astype(np.float64),
             quats=sc.quats.astype(np.float64) * (1.7 if rotated else 1.0),
             opacity=sc.opacity.astype(np.float64), colors=sc.colors.astype(np.float64))
    return cam, P, sc.dL_dimage[0].astype(np.float64)


@pytest.mark.parametrize("seed,rotated", [(1, False), (3, True)])
def test_gradients_match_central_differences(seed, rotated):
    cam, P, g = _fd_scene(seed, rotated)

    def loss(Q):
        f = oracle.forward(cam, Q["means"], Q["scales"], Q["quats"], Q["opacity"], Q["colors"], "f64")
        return float((f["image"] * g).sum())

    fb = oracle.forward_backward(cam, P["means"], P["scales"], P["quats"], P["opacity"], P["colors"], g, "f64")
    assert np.all(fb["pre"]["radius"] > 0)
    eps = 1e-4
    names = dict(means="dL_dmeans", scales="dL_dscales", quats="dL_dquats", opacity="dL_dopacity",
                 colors="dL_dcolors")
    for k, gk in names.items():
        fd = np.zeros_like(P[k])
        for i in range(P[k].size):
            Qp = {kk: v.copy() for kk, v in P.items()}
            Qm = {kk: v.copy() for kk, v in P.items()}
            Qp[k].reshape(-1)[i] += eps
            Qm[k].reshape(-1)[i] -= eps
            fd.reshape(-1)[i] = (loss(Qp) - loss(Qm)) / (2 * eps)
        scale = np.abs(fd).max()
        assert scale > 0
        np.testing.assert_allclose(fb[gk], fd, atol=1e-5 * scale, rtol=0, err_msg=k)


def test_opacity_cap_gradient_is_exact_zero():
    """When sigma G > 0.99 the cap is active: alpha does not depend on sigma or
    G, so the exact derivative w.r.t. opacity and the conic is zero."""
    cam = _cam(32, 32, 32.0, sigma_mult=50.0, alpha_min=0.0, T_min=0.0)
    f = oracle.forward_backward(cam, [[0.03125, 0.03125, 2.0]], _iso(1, 0.5), _ident_q(1), [1.0], [[1, 0.5, 0.2]],
                                np.zeros((3, 32, 32)) + 1.0, "f64")
    # only pixels where 1.0 * G <= 0.99 contribute; compare with the sum over them
    assert f["dL_dopacity"][0] != 0.0
    g = np.zeros((3, 32, 32))
    g[:, 16, 16] = 1.0  # pixel at the mean: G = 1, capped
    f1 = oracle.forward_backward(cam, [[0.03125, 0.03125, 2.0]], _iso(1, 0.5), _ident_q(1), [1.0], [[1, 0.5, 0.2]],
                                 g, "f64")
    assert f1["dL_dopacity"][0] == 0.0
    assert not f1["dL_dconic_opacity"][0, :3].any() and not f1["dL_dmean2d"].any()


def test_isotropic_scales_give_zero_quaternion_gradient():
    sc = scenes.random_tiny(n=6, seed=4)
    s = np.repeat(sc.scales[:, :1], 3, axis=1).astype(np.float64)
    fb = oracle.forward_backward(sc.cameras[0], sc.means, s, sc.quats, sc.opacity, sc.colors, sc.dL_dimage[0], "f64")
    assert np.abs(fb["dL_dscales"]).max() > 0
    assert np.abs(fb["dL_dquats"]).max() < 1e-12 * np.abs(fb["dL_dscales"]).max()


def test_quaternion_gradient_orthogonal_to_q_and_scale_covariant():
    sc = scenes.random_tiny(n=6, seed=5)
    q = sc.quats.astype(np.float64)
    a = oracle.forward_backward(sc.cameras[0], sc.means, sc.scales, q, sc.opacity, sc.colors, sc.dL_dimage[0], "f64")
    b = oracle.forward_backward(sc.cameras[0], sc.means, sc.scales, 2 * q, sc.opacity, sc.colors, sc.dL_dimage[0],
                                "f64")
    np.testing.assert_allclose(a["image"], b["image"], atol=1e-12)
    dq = a["dL_dquats"]
    assert np.abs((dq * q).sum(1)).max() < 1e-12 * np.abs(dq).max()
    np.testing.assert_allclose(b["dL_dquats"], 0.5 * dq, atol=1e-12 * np.abs(dq).max())


@pytest.mark.parametrize("thresholds", [(0.0, 0.0), (1 / 255, 1e-4)])
def test_colour_gradient_sums_to_coverage(thresholds):
    """C is linear in the colours with weights alpha_k T_k summing to
    1 - T_final, so sum over Gaussians of dL/dc = sum over pixels of
    (1 - T_final) dL/dC, per channel."""
    sc = scenes.preset(1)
    cam = sc.cameras[0].replace(alpha_min=thresholds[0], T_min=thresholds[1])
    g = sc.dL_dimage[0].astype(np.float64)
    fb = oracle.forward_backward(cam, sc.means, sc.scales, sc.quats, sc.opacity, sc.colors, g, "f64")
    lhs = fb["dL_dcolor"].sum(0)
    rhs = ((1 - fb["final_T"])[None] * g).sum((1, 2))
    np.testing.assert_allclose(lhs, rhs, rtol=1e-10)


def test_conic_gradient_matches_covariance_closed_form():
    """For one pixel, d G / d Sigma2 = 1/2 G Sigma2^-1 d d^T Sigma2^-1 (the
    Gaussian-PDF gradient of the page '3D高斯前向传播与反向传播原理详解' without
    its normaliser term).  The oracle's conic gradient, taken to Sigma2 through
    d(A^-1) = -A^-1 dA A^-1, must equal dL/dG times that."""
    cam = _cam(32, 32, 32.0, sigma_mult=50.0, alpha_min=0.0, T_min=0.0, bg=(0.0, 0.0, 0.0))
    mu = [[0.05, -0.04, 2.5]]
    sc = [[0.06, 0.1, 0.08]]
    q = [[0.9, 0.2, -0.3, 0.1]]
    sig, col = 0.6, [0.7, 0.2, 0.4]
    px, py = 20, 13
    g = np.zeros((3, 32, 32))
    g[:, py, px] = [0.3, -0.8, 0.5]
    fb = oracle.forward_backward(cam, mu, sc, q, [sig], [col], g, "f64")
    u, v = fb["pre"]["mean2d"][0]
    a, b, c, _ = fb["pre"]["conic_opacity"][0]
    A = np.array([[a, b], [b, c]])
    d = np.array([px + 0.5 - u, py + 0.5 - v])
    G = math.exp(-0.5 * d @ A @ d)
    dL_dG = sig * float(np.dot(col, g[:, py, px]))  # bg = 0 and one Gaussian: C = sigma G c
    expected = dL_dG * 0.5 * G * (A @ np.outer(d, d) @ A)
    ga, gb, gc, _ = fb["dL_dconic_opacity"][0]
    GA = np.array([[ga, 0.5 * gb], [0.5 * gb, gc]])
    got = -A @ GA @ A
    np.testing.assert_allclose(got, expected, rtol=1e-10, atol=1e-14)
    # and the 2D mean gradient has the sign of dG/dmu = G A (x - mu)
    np.testing.assert_allclose(fb["dL_dmean2d"][0], dL_dG * G * (A @ d), rtol=1e-10)


def test_culled_gaussians_get_zero_gradient():
    cam = _cam(32, 32, 32.0)
    means = [[0, 0, 3.0], [0, 0, 0.05], [50, 0, 3.0]]
    g = np.random.default_rng(0).normal(size=(3, 32, 32))
    fb = oracle.forward_backward(cam, means, _iso(3, 0.05), _ident_q(3), [0.5] * 3, [[1, 1, 1]] * 3, g, "f64")
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors"):
        assert not np.asarray(fb[k])[1:].any(), k
    assert np.abs(fb["dL_dmeans"][0]).max() > 0


def test_backward_is_deterministic_across_thread_counts():
    sc = scenes.preset(2)
    cam = sc.cameras[0]
    n0 = oracle.num_threads()
    try:
        oracle.set_threads(1)
        a = oracle.forward_backward(cam, sc.means, sc.scales, sc.quats, sc.opacity, sc.colors, sc.dL_dimage[0], "f64")
        oracle.set_threads(max(2, n0))
        b = oracle.forward_backward(cam, sc.means, sc.scales, sc.quats, sc.opacity, sc.colors, sc.dL_dimage[0], "f64")
    finally:
        oracle.set_threads(n0)
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors"):
        np.testing.assert_array_equal(a[k], b[k])


def test_mirror_exp_error_bound():
    """The fp32 mirror's exp (a fixed IEEE sequence that the kernels repeat
    bit for bit) is within 2 ulp of exp over the range compositing uses."""
    x = np.concatenate([np.linspace(-87.0, 0.0, 2_000_001, dtype=np.float32),
                        np.float32(-np.logspace(-8, 1.9, 200_001)),
                        np.array([0.0, -0.0, -1e-30, -87.0, -100.0, -np.inf], np.float32)])
    y = oracle.exp_f32(x)
    ref = np.exp(np.maximum(x.astype(np.float64), -87.0))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    err = np.abs(y.astype(np.float64) - ref) / ulp
    assert err.max() <= 2.0, err.max()
    assert oracle.exp_f32(np.zeros(1))[0] == 1.0


def test_densification_statistics_closed_form():
    """The densification accumulator of one isotropic Gaussian on the optical
    axis, seen by two identical views and by a third that culls it, equals
    twice the norm of the hand-derived 2D mean gradient.  With one Gaussian,
    alpha = sigma G (no cap, no thresholds), C = alpha c + (1 - alpha) bg, and
    an upstream gradient of 1 on channel 0 of one pixel p0, the mean gradient
    of the chain-rule page (dG/dmu = G Sigma^-1 (x - mu)) gives
    dL/dmean2d = (c_0 - bg_0) sigma G(p0) (p0 - mu) / s2^2 with
    s2^2 = (f s / z)^2 + eps."""
    f, z, s, sig = 32.0, 3.0, 0.2, 0.8
    cam = _cam(32, 32, f, sigma_mult=50.0, alpha_min=0.0, T_min=0.0, bg=(0.1, 0.2, 0.3))
    col = [0.9, 0.4, 0.6]
    x0, y0 = 19, 14
    dl = np.zeros((3, 32, 32))
    dl[0, y0, x0] = 1.0
    means, scales, quats = np.array([[0.0, 0.0, z]]), np.array([[s, s, s]]), _ident_q(1)
    s22 = (f * s / z) ** 2 + _f32(cam.eps2d)
    d = np.array([x0 + 0.5 - 16.0, y0 + 0.5 - 16.0])
    G = math.exp(-(d @ d) / (2.0 * s22))
    expect = (col[0] - _f32(cam.bg[0])) * sig * G * d / s22
    behind = cam.replace(t=(0.0, 0.0, -10.0))  # the Gaussian is behind this camera: culled
    out = None
    for c in (cam, behind, cam):
        fb = oracle.forward_backward(c, means, scales, quats, [sig], [col], dl, "f64")
        if c is cam:
            np.testing.assert_allclose(fb["dL_dmean2d"][0], expect, rtol=1e-10)
        out = oracle.preprocess_bwd(c, means, scales, quats, fb["pre"]["radius"], fb["dL_dmean2d"],
                                    fb["dL_dconic_opacity"], fb["dL_dcolor"], "f64", accumulate_into=out,
                                    densify=True)
    assert out["grad2d_accum"][0] == pytest.approx(2.0 * float(np.linalg.norm(expect)), rel=1e-10)
    assert out["vis_count"][0] == 2
