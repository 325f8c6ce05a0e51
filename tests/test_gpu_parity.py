"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars: bit-exact preprocess integers, depth bits, tile ranges, sorted ids and
64-bit keys; contributor counts equal on >= 99.99% of pixels; image absolute
error <= 1e-4; per-tensor gradient relative L2 error <= 1e-3 (fp32 kernels
against the float64 oracle).
"""
import numpy as np
import pytest
import torch

import oracle
from differentiable_gaussian_splatting_preprocess_b200 import binding as B
from differentiable_gaussian_splatting_preprocess_b200 import scenes

from _gpu_pipeline import (GRAD_REL_L2, IMAGE_ATOL, N_CONTRIB_MATCH, GpuScene, frame_np, rel_l2, run_gpu, to_dev,
                           to_np)

pytestmark = pytest.mark.gpu

_CACHE = {}


def _scene(cfg):
    if cfg not in _CACHE:
        _CACHE.clear()
        _CACHE[cfg] = scenes.preset(cfg)
    return _CACHE[cfg]


def _check_preprocess(sc, cam, g):
    o = oracle.preprocess(cam, sc.means, sc.scales, sc.quats, sc.opacity, "f32")
    for k in ("radius", "rect", "tiles_touched"):
        np.testing.assert_array_equal(g[k], o[k], err_msg=k)
    for k in ("depth", "mean2d", "conic_opacity"):
        np.testing.assert_array_equal(g[k].view(np.uint32), o[k].view(np.uint32), err_msg=k)
    assert g["num_pairs"] == int(o["tiles_touched"].astype(np.uint64).sum())
    return o


def _check_bins(cam, g, pre):
    b = oracle.bin_pairs(cam, pre["depth"], pre["rect"], pre["tiles_touched"], "f32")
    assert b["num_pairs"] == g["num_pairs"]
    np.testing.assert_array_equal(g["ranges"], b["ranges"])
    np.testing.assert_array_equal(g["ids"], b["ids"])
    np.testing.assert_array_equal(g["keys"], b["keys"])
    return b


def _check_render_fwd(cam, sc, g, tiles=None):
    o = oracle.render_fwd(cam, g["ranges"], g["ids"], g["mean2d"], g["conic_opacity"], sc.colors, "f32", tiles=tiles)
    if tiles is None:
        mask = np.ones((cam.height, cam.width), bool)
    else:
        mask = np.zeros((cam.height, cam.width), bool)
        TX = cam.tiles_x
        for t in tiles:
            tx, ty = t % TX, t // TX
            mask[ty * 16:(ty + 1) * 16, tx * 16:(tx + 1) * 16] = True
    err = np.abs(g["image"] - o["image"])[:, mask].max()
    assert err <= IMAGE_ATOL, f"image abs err {err}"
    match = (g["n_contrib"][mask] == o["n_contrib"][mask]).mean()
    assert match >= N_CONTRIB_MATCH, f"n_contrib match {match}"
    assert np.abs(g["final_T"] - o["final_T"])[mask].max() <= IMAGE_ATOL
    # Stronger than the bar: alpha, the skip and stop decisions and T are
    # computed by the same fixed IEEE steps on both sides (the quadratic form
    # with explicit fused multiply-adds and the shared exp sequence), so the
    # contributor counts and the final transmittance agree bit for bit.
    np.testing.assert_array_equal(g["n_contrib"][mask], o["n_contrib"][mask])
    np.testing.assert_array_equal(g["final_T"][mask].view(np.uint32), o["final_T"][mask].view(np.uint32))
    return o


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_forward_parity(cfg):
    sc = _scene(cfg)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    r = run_gpu(gs, cam)
    g = frame_np(r["frame"])
    assert r["rz"].status() == 0
    pre = _check_preprocess(sc, cam, g)
    _check_bins(cam, g, pre)          # isolated == end to end: preprocess is bit-exact
    _check_render_fwd(cam, sc, g)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_backward_parity(cfg):
    sc = _scene(cfg)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    r = run_gpu(gs, cam, dL_dimage=sc.dL_dimage[0])
    g = frame_np(r["frame"])
    gr = {k: to_np(v) for k, v in r["grads"].items()}
    # 2D gradients on identical inputs (isolated)
    o2 = oracle.render_bwd(cam, sc.N, g["ranges"], g["ids"], g["mean2d"], g["conic_opacity"], sc.colors,
                           sc.dL_dimage[0], "f64")
    assert rel_l2(gr["dL_dmean2d"], o2["dL_dmean2d"]) <= GRAD_REL_L2
    assert rel_l2(gr["dL_dconic_opacity"][:, :3], o2["dL_dconic_opacity"][:, :3]) <= GRAD_REL_L2
    assert rel_l2(gr["dL_dconic_opacity"][:, 3], o2["dL_dconic_opacity"][:, 3]) <= GRAD_REL_L2
    assert rel_l2(gr["dL_dcolor"], o2["dL_dcolor"]) <= GRAD_REL_L2
    # 3D gradients from the same 2D gradients (isolated chain rule)
    o3 = oracle.preprocess_bwd(cam, sc.means, sc.scales, sc.quats, g["radius"], gr["dL_dmean2d"],
                               gr["dL_dconic_opacity"], gr["dL_dcolor"], "f64")
    # (tighter than the acceptance bar: an fp32 chain of ~100 operations)
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors"):
        e = rel_l2(gr[k], o3[k])
        assert e <= 1e-4, (k, e)
    # end to end: the float64 oracle's own forward and backward (its own
    # projection, binning and compositing decisions, rounded independently)
    f = oracle.forward_backward(cam, sc.means, sc.scales, sc.quats, sc.opacity, sc.colors, sc.dL_dimage[0], "f64")
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors"):
        e = rel_l2(gr[k], f[k])
        assert e <= GRAD_REL_L2, (k, e)
    _check_against_f64(cam, sc, g, f, r["frame"])


def _check_against_f64(cam, sc, g, f_e2e, fr, tiles=None, mask=None):
    """Against float64, rounded independently of the kernels (std::exp,
    double products):
    * compositing decisions: the float64 compositing of the GPU's own lists
      and 2D records (the same inputs, so the only difference is the
      arithmetic) gives the same contributor counts (last contributor) on
      >= 99.99% of pixels and the same image within 1e-4 on >= 99.99%;
    * end to end, the float64 pipeline (its own projection and binning as
      well): the image within 1e-4 on >= 99.99% of pixels; the number of
      terms blended per pixel agrees on >= 99.9% (the float64 projection
      rounds the conics and a few tile rectangles differently, which moves
      alpha_min and T_min decisions at about 2e-4 of the pixels of the 1M
      scene; integer decisions are held to the 99.99% bar in equal inputs)."""
    if mask is None:
        mask = np.ones(g["n_contrib"].shape, bool)
    iso = oracle.render_fwd(cam, g["ranges"], g["ids"], g["mean2d"].astype(np.float64),
                            g["conic_opacity"].astype(np.float64), sc.colors, "f64", tiles=tiles)
    match = (g["n_contrib"][mask] == iso["n_contrib"][mask]).mean()
    assert match >= N_CONTRIB_MATCH, f"n_contrib match vs float64 compositing {match}"
    bad = (np.abs(g["image"] - iso["image"]) > IMAGE_ATOL).any(0)[mask].mean()
    assert bad <= 1.0 - N_CONTRIB_MATCH, f"image pixels beyond {IMAGE_ATOL} vs float64 compositing: {bad}"
    bad = (np.abs(g["image"] - f_e2e["image"]) > IMAGE_ATOL).any(0)[mask].mean()
    assert bad <= 1.0 - N_CONTRIB_MATCH, f"image pixels beyond {IMAGE_ATOL} vs float64 pipeline: {bad}"
    ne = torch.empty((cam.height, cam.width), dtype=torch.uint32, device="cuda")
    nb = torch.empty_like(ne)
    B.gs_render_stats(cam, fr.ranges, fr.ids, fr.mean2d, fr.conic_opacity, ne, nb)
    torch.cuda.synchronize()
    match = (to_np(nb)[mask] == f_e2e["n_blended"][mask]).mean()
    assert match >= 0.999, f"blended-term count match vs float64 pipeline {match}"


def _sample_tiles(cam, n, seed):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(cam.num_tiles, size=min(n, cam.num_tiles), replace=False)).astype(np.int32)


@pytest.mark.slow
def test_config5_four_cameras():
    """3M Gaussians, four cameras rendered back to back with 3D gradients
    accumulated.  Per camera: preprocess bit-exact; every tile range and every
    tile's sorted id list bit-exact against the oracle's binning; every tile
    composited against the fp32 mirror (image, final T, contributor counts);
    sampled tiles' image and contributor counts against the float64 pipeline;
    sampled tiles' gradients against the float64 oracle (the upstream gradient
    is restricted to the sampled tiles, so the oracle's backward only has to
    run those)."""
    sc = _scene(5)
    gs = GpuScene(sc)
    grads = None
    o3 = None
    for ci, cam in enumerate(sc.cameras):
        tiles = _sample_tiles(cam, 12, ci)
        mask = np.zeros((cam.height, cam.width), bool)
        for t in tiles:
            tx, ty = t % cam.tiles_x, t // cam.tiles_x
            mask[ty * 16:(ty + 1) * 16, tx * 16:(tx + 1) * 16] = True
        dl = np.where(mask[None], sc.dL_dimage[ci], 0.0).astype(np.float32)
        r = run_gpu(gs, cam, dL_dimage=dl, want_keys=False, grads=grads)
        assert r["rz"].status() == 0
        grads = {k: r["grads"][k] for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors")}
        g = frame_np(r["frame"])
        pre = _check_preprocess(sc, cam, g)
        b = oracle.bin_pairs(cam, pre["depth"], pre["rect"], pre["tiles_touched"], "f32", want_keys=False)
        assert b["num_pairs"] == g["num_pairs"]
        np.testing.assert_array_equal(g["ranges"], b["ranges"])
        np.testing.assert_array_equal(g["ids"], b["ids"])
        del b
        for t in tiles[:3]:  # the per-tile brute force, independent of the oracle's grouping
            s, e = g["ranges"][t]
            np.testing.assert_array_equal(g["ids"][s:e], oracle.tile_list(cam, pre["depth"], pre["rect"],
                                                                          pre["tiles_touched"], int(t)))
        _check_render_fwd(cam, sc, g)
        f64 = oracle.forward(cam, sc.means, sc.scales, sc.quats, sc.opacity, sc.colors, "f64")
        _check_against_f64(cam, sc, g, f64, r["frame"])
        del f64
        o2 = oracle.render_bwd(cam, sc.N, g["ranges"], g["ids"], g["mean2d"], g["conic_opacity"], sc.colors, dl,
                               "f64", tiles=tiles)
        gr = {k: to_np(r["grads"][k]) for k in ("dL_dmean2d", "dL_dconic_opacity", "dL_dcolor")}
        assert rel_l2(gr["dL_dmean2d"], o2["dL_dmean2d"]) <= GRAD_REL_L2
        assert rel_l2(gr["dL_dconic_opacity"], o2["dL_dconic_opacity"]) <= GRAD_REL_L2
        assert rel_l2(gr["dL_dcolor"], o2["dL_dcolor"]) <= GRAD_REL_L2
        o3 = oracle.preprocess_bwd(cam, sc.means, sc.scales, sc.quats, g["radius"], o2["dL_dmean2d"],
                                   o2["dL_dconic_opacity"], o2["dL_dcolor"], "f64", accumulate_into=o3)
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors"):
        e = rel_l2(to_np(grads[k]), o3[k])
        assert e <= GRAD_REL_L2, (k, e)


# --------------------------------------------------------------------------
# Edge cases
# --------------------------------------------------------------------------

def _tiny(**kw):
    return scenes.random_tiny(**kw)


def test_empty_scene():
    cam = scenes.Camera(40, 24, 40.0, 40.0, 20.0, 12.0, bg=(0.25, 0.5, 0.75))
    e = np.zeros((0, 3), np.float32)
    sc = scenes.Scene("empty", e, e, np.zeros((0, 4), np.float32), np.zeros(0, np.float32), e, [cam],
                      [np.ones((3, 24, 40), np.float32)])
    gs = GpuScene(sc)
    r = run_gpu(gs, cam, dL_dimage=sc.dL_dimage[0], want_keys=True)
    g = frame_np(r["frame"])
    assert g["num_pairs"] == 0 and not g["ranges"].any()
    np.testing.assert_array_equal(g["image"], np.broadcast_to(np.array([0.25, 0.5, 0.75], np.float32)[:, None, None],
                                                              (3, 24, 40)))
    assert np.all(g["final_T"] == 1.0) and not g["n_contrib"].any()


def test_all_culled():
    sc = _tiny(n=20, seed=3)
    sc.means[:, 2] = -1.0
    gs = GpuScene(sc)
    r = run_gpu(gs, sc.cameras[0], dL_dimage=sc.dL_dimage[0])
    g = frame_np(r["frame"])
    assert g["num_pairs"] == 0 and not g["radius"].any()
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors"):
        assert not to_np(r["grads"][k]).any()


@pytest.mark.parametrize("W,H", [(37, 23), (16, 16), (1, 1), (300, 17)])
def test_ragged_and_tiny_images(W, H):
    sc = _tiny(n=40, width=W, height=H, seed=W + H, z_range=(1.5, 6.0))
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    dl = np.random.default_rng(0).normal(size=(3, H, W)).astype(np.float32)
    r = run_gpu(gs, cam, dL_dimage=dl)
    g = frame_np(r["frame"])
    pre = _check_preprocess(sc, cam, g)
    _check_bins(cam, g, pre)
    _check_render_fwd(cam, sc, g)
    f = oracle.forward_backward(cam, sc.means, sc.scales, sc.quats, sc.opacity, sc.colors, dl, "f64")
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors"):
        assert rel_l2(to_np(r["grads"][k]), f[k]) <= GRAD_REL_L2, k


@pytest.mark.parametrize("W,H,n,sigma_mult", [(16400, 20, 80, 3.0), (8200, 40, 80, 3.0), (40, 8200, 80, 3.0),
                                              (800, 608, 2000, 1e3), (2000, 1200, 300, 3.0), (2000, 2100, 200, 3.0),
                                              (8200, 600, 80, 3.0)])
def test_binning_routes(W, H, n, sigma_mult):
    """Both binning routes against the oracle's sort: more than 1024 tile
    columns (257 cells: emit + radix sort by tile id + boundary ranges),
    129 cell columns or rows (cell passes with 8-bit digits), cell pairs of
    whole-image Gaussians cut by every chunk boundary of the generated first
    pass, and larger cell grids (32 x 19, 32 x 33, 129 x 10 cells)."""
    sc = _tiny(n=n, width=W, height=H, seed=W + 3 * H, z_range=(2.0, 6.0), sigma_mult=sigma_mult)
    cam = sc.cameras[0].replace(fx=float(W), fy=float(H), cx=W / 2.0, cy=H / 2.0)
    sc.cameras[0] = cam
    gs = GpuScene(sc)
    g = frame_np(run_gpu(gs, cam)["frame"])
    pre = _check_preprocess(sc, cam, g)
    assert g["num_pairs"] > 0
    _check_bins(cam, g, pre)


def test_rank_scan_over_more_than_2048_blocks():
    """5M Gaussians: the rank-order scan has 2442 blocks, so each block of
    its second kernel sums the per-block partials below it in two rounds
    (2048 per round); the depth sort runs at its maximum grid with several
    tiles per CTA.  Preprocess and binning against the oracle, bit-exact."""
    sc = _tiny(n=5_000_000, width=256, height=256, seed=11, distinct_depth_gap=None, scale_log_mean=-4.0)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    g = frame_np(run_gpu(gs, cam)["frame"])
    pre = _check_preprocess(sc, cam, g)
    assert g["num_pairs"] > 0
    _check_bins(cam, g, pre)


def test_no_thresholds_and_large_support():
    """alpha_min = T_min = 0 and a support radius covering the whole image."""
    sc = _tiny(n=24, width=64, height=48, seed=11, sigma_mult=1e3, alpha_min=0.0, T_min=0.0)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    r = run_gpu(gs, cam, dL_dimage=sc.dL_dimage[0])
    g = frame_np(r["frame"])
    pre = _check_preprocess(sc, cam, g)
    assert np.all(pre["tiles_touched"] == cam.num_tiles)
    _check_bins(cam, g, pre)
    _check_render_fwd(cam, sc, g)
    f = oracle.forward_backward(cam, sc.means, sc.scales, sc.quats, sc.opacity, sc.colors, sc.dL_dimage[0], "f64")
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors"):
        assert rel_l2(to_np(r["grads"][k]), f[k]) <= GRAD_REL_L2, k


def test_capacity_overflow_is_reported_and_recoverable():
    sc = _scene(2)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    r = run_gpu(gs, cam, capacity=1000)
    rz = r["rz"]
    assert rz.status() & B.GS_ERR_CAPACITY
    assert not to_np(r["frame"].ranges).any()
    B.gs_clear_status(rz.ws)
    assert rz.status() == 0
    fr = rz.forward(gs.means, gs.scales, gs.quats, gs.opacity, gs.colors)
    torch.cuda.synchronize()
    assert rz.status() == 0 and int(to_np(fr.num_pairs)[0]) > 1000


def test_pair_count_overflow_is_reported():
    """A 65536 x 65536 image (4096 x 4096 tiles) with 300 Gaussians whose
    support covers it: 300 * 2^24 pairs exceed 2^32 - 1.  The preprocess
    reports GS_ERR_OVERFLOW, saturates the device pair count, and a binning
    call then reports the capacity error and leaves every range empty."""
    sc = _tiny(n=300, width=64, height=64, seed=9, sigma_mult=1e4)
    cam = sc.cameras[0].replace(width=65536, height=65536, fx=65536.0, fy=65536.0, cx=32768.0, cy=32768.0)
    gs = GpuScene(sc)
    from differentiable_gaussian_splatting_preprocess_b200 import rasterizer as RZ
    rz = RZ.Rasterizer(cam)
    pre = rz.preprocess(gs.means, gs.scales, gs.quats, gs.opacity)
    torch.cuda.synchronize()
    tt = to_np(pre["tiles_touched"]).astype(np.int64)
    o = oracle.preprocess(cam, sc.means, sc.scales, sc.quats, sc.opacity, "f32")
    np.testing.assert_array_equal(tt, o["tiles_touched"])
    assert tt.sum() > 0xFFFFFFFF and tt.max() == 4096 * 4096
    assert rz.status() & B.GS_ERR_OVERFLOW
    assert int(to_np(pre["num_pairs"]).view(np.uint32)[0]) == 0xFFFFFFFF
    ids = torch.empty(1000, dtype=torch.uint32, device="cuda")
    ranges = torch.full((B.num_tiles(cam), 2), 7, dtype=torch.uint32, device="cuda")
    B.gs_bin_sort(cam, pre["depth"], pre["rect"], pre["tiles_touched"], pre["num_pairs"], 1000, ids, ranges, None,
                  rz.workspace(sc.N, 1000))
    torch.cuda.synchronize()
    assert rz.status() & B.GS_ERR_CAPACITY
    assert not to_np(ranges).any()
    B.gs_clear_status(rz.ws)
    assert rz.status() == 0


def test_capacity_mode_matches_host_sized():
    sc = _scene(2)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    a = frame_np(run_gpu(gs, cam)["frame"])
    b = frame_np(run_gpu(gs, cam, capacity=a["num_pairs"] + 12345)["frame"])
    for k in ("ranges", "ids", "keys", "image", "n_contrib"):
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_degenerate_inputs_are_culled():
    sc = _tiny(n=8, seed=5)
    sc.means[0] = np.nan
    sc.quats[1] = 0.0
    sc.scales[2] = 0.0  # zero covariance: dilation keeps the determinant positive
    sc.means[3, 2] = 0.1  # nearer than z_near
    gs = GpuScene(sc)
    r = run_gpu(gs, sc.cameras[0], dL_dimage=sc.dL_dimage[0])
    g = frame_np(r["frame"])
    pre = _check_preprocess(sc, sc.cameras[0], g)
    assert list(pre["radius"][[0, 1, 3]]) == [0, 0, 0]
    assert pre["radius"][2] > 0
    _check_render_fwd(sc.cameras[0], sc, g)
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats"):
        v = to_np(r["grads"][k])
        assert np.all(np.isfinite(v)) and not v[[0, 1, 3]].any()


def test_invalid_arguments_raise_without_launch():
    sc = _tiny(n=4)
    gs = GpuScene(sc)
    cam = sc.cameras[0]
    bad = cam.replace(tile=8)
    from differentiable_gaussian_splatting_preprocess_b200 import rasterizer as RZ
    with pytest.raises(B.GsError):
        RZ.Rasterizer(bad).forward(gs.means, gs.scales, gs.quats, gs.opacity, gs.colors)
    rz = RZ.Rasterizer(cam)
    small_ws = torch.zeros(16, dtype=torch.uint8, device="cuda")
    out = rz.preprocess(gs.means, gs.scales, gs.quats, gs.opacity)
    with pytest.raises(B.GsError):
        B.gs_preprocess_fwd(cam, gs.means, gs.scales, gs.quats, gs.opacity, out["mean2d"], out["depth"],
                            out["conic_opacity"], out["radius"], out["rect"], out["tiles_touched"],
                            out["num_pairs"], small_ws)


def test_preprocess_backward_accumulates():
    sc = _tiny(n=16, seed=9)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    r1 = run_gpu(gs, cam, dL_dimage=sc.dL_dimage[0])
    once = {k: to_np(v).copy() for k, v in r1["grads"].items()}
    r2 = run_gpu(gs, cam, dL_dimage=sc.dL_dimage[0], grads={k: v.clone() for k, v in r1["grads"].items()
                                                              if k.startswith("dL_d") and v.shape[0] == sc.N})
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors"):
        np.testing.assert_allclose(to_np(r2["grads"][k]), 2 * once[k], rtol=1e-5, atol=1e-7)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_render_stats_match_oracle_counts(cfg):
    """The work counts behind the throughput figures (entries evaluated and
    terms blended per pixel) equal the oracle's, bit for bit."""
    sc = _scene(cfg)
    cam = sc.cameras[0]
    r = run_gpu(GpuScene(sc), cam, want_keys=False)
    fr = r["frame"]
    ne = torch.empty((cam.height, cam.width), dtype=torch.uint32, device="cuda")
    nb = torch.empty_like(ne)
    B.gs_render_stats(cam, fr.ranges, fr.ids, fr.mean2d, fr.conic_opacity, ne, nb)
    torch.cuda.synchronize()
    g = frame_np(fr)
    o = oracle.render_fwd(cam, g["ranges"], g["ids"], g["mean2d"], g["conic_opacity"], sc.colors, "f32")
    np.testing.assert_array_equal(to_np(ne), o["n_eval"])
    np.testing.assert_array_equal(to_np(nb), o["n_blended"])
    assert np.all(to_np(nb) <= g["n_contrib"])


def _work_class(w: np.ndarray) -> np.ndarray:
    """The render's 8-bit dispatch class: exact below 16, then 8 classes per octave."""
    w = w.astype(np.int64)
    e = np.floor(np.log2(np.maximum(w, 1))).astype(np.int64)
    return np.where(w < 16, w, 16 + (e - 4) * 8 + ((w >> np.maximum(e - 3, 0)) & 7))


def _check_dispatch_order(mask: np.ndarray, ranges: np.ndarray, blend_mask: np.ndarray) -> None:
    """The dispatch-order block after a forward and a backward with the mask:
    per quadrant the number of its blended positions (from the oracle's
    contribution bits), the forward's tile order (a permutation of the tiles
    in decreasing class of list length) and the backward's quadrant order (a
    permutation of the quadrants in decreasing class of those counts)."""
    T = ranges.shape[0]
    rg = ranges.astype(np.int64)
    L = rg[:, 1] - rg[:, 0]
    k = np.concatenate([np.arange(a, b) for a, b in rg if b > a]) if L.sum() else np.zeros(0, np.int64)
    tile_of = np.repeat(np.arange(T), L)
    words = blend_mask.reshape(-1, 4)
    want_work = np.zeros((T, 4), np.int64)
    for q in range(4):
        bit = (words[k >> 5, q] >> (k & 31).astype(np.uint32)) & 1
        want_work[:, q] = np.bincount(tile_of, weights=bit, minlength=T).astype(np.int64)
    quad_work = mask[:4 * T].astype(np.int64)
    np.testing.assert_array_equal(quad_work, want_work.reshape(-1))
    for order, work in ((mask[4 * T:8 * T].astype(np.int64), quad_work), (mask[8 * T:9 * T].astype(np.int64), L)):
        np.testing.assert_array_equal(np.sort(order), np.arange(work.size))
        assert np.all(np.diff(_work_class(work[order])) <= 0)


@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_contribution_mask_and_backward_without_it(cfg):
    """The forward's per-quadrant contribution mask equals the oracle's bit for
    bit, the dispatch-order block holds the per-quadrant counts and the two
    heaviest-first orders, and the backward gives the same gradients with and
    without the mask."""
    sc = _scene(cfg)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    r = run_gpu(gs, cam, dL_dimage=sc.dL_dimage[0], want_keys=False)
    fr = r["frame"]
    g = frame_np(fr)
    P = g["num_pairs"]
    o = oracle.render_fwd(cam, g["ranges"], g["ids"], g["mean2d"], g["conic_opacity"], sc.colors, "f32",
                          blend_mask=True)
    words = 4 * ((P + 31) // 32)
    ow = B.order_words(B.num_tiles(cam))
    np.testing.assert_array_equal(to_np(fr.contrib_mask)[ow:ow + words], o["blend_mask"][:words])
    _check_dispatch_order(to_np(fr.contrib_mask), g["ranges"], o["blend_mask"])
    with_mask = {k: to_np(r["grads"][k]).copy() for k in ("dL_dmean2d", "dL_dconic_opacity", "dL_dcolor")}
    outs = {k: torch.empty_like(r["grads"][k]) for k in with_mask}
    B.gs_render_bwd(cam, fr.ranges, fr.ids, fr.mean2d, fr.conic_opacity, gs.colors, fr.final_T, fr.n_contrib,
                    to_dev(sc.dL_dimage[0]), outs["dL_dmean2d"], outs["dL_dconic_opacity"], outs["dL_dcolor"], None)
    torch.cuda.synchronize()
    for k in with_mask:
        assert rel_l2(to_np(outs[k]), with_mask[k]) <= 1e-5, k


def test_densification_statistics_over_views():
    """The statistics accumulated over the four cameras of the 3M scene equal
    the oracle's (gradients restricted to sampled tiles keep the oracle fast)."""
    sc = _scene(3)
    cams = [sc.cameras[0], sc.cameras[0].replace(R=(0.985, 0.0, 0.174, 0.0, 1.0, 0.0, -0.174, 0.0, 0.985))]
    gs = GpuScene(sc)
    dens = dict(grad2d_accum=torch.zeros(sc.N, device="cuda"),
                vis_count=torch.zeros(sc.N, dtype=torch.uint32, device="cuda"))
    out = None
    from differentiable_gaussian_splatting_preprocess_b200 import rasterizer as RZ
    for cam in cams:
        rz = RZ.Rasterizer(cam)
        fr = rz.forward(gs.means, gs.scales, gs.quats, gs.opacity, gs.colors)
        g = rz.backward(fr, gs.means, gs.scales, gs.quats, gs.colors, to_dev(sc.dL_dimage[0]), densify=dens)
        torch.cuda.synchronize()
        out = oracle.preprocess_bwd(cam, sc.means, sc.scales, sc.quats, to_np(fr.radius), to_np(g["dL_dmean2d"]),
                                    to_np(g["dL_dconic_opacity"]), to_np(g["dL_dcolor"]), "f64",
                                    accumulate_into=out, densify=True)
    np.testing.assert_array_equal(to_np(dens["vis_count"]), out["vis_count"])
    assert rel_l2(to_np(dens["grad2d_accum"]), out["grad2d_accum"]) <= 1e-6


def test_render_views_sums_cameras():
    """Several views rendered back to back with the 3D gradients summed equal
    the sum of the oracle's per-view gradients."""
    from differentiable_gaussian_splatting_preprocess_b200 import multiview as MV
    sc = _scene(2)
    base = sc.cameras[0]
    cams = [base, base.replace(R=(0.985, 0.0, 0.174, 0.0, 1.0, 0.0, -0.174, 0.0, 0.985)),
            base.replace(t=(0.2, -0.1, 0.0))]
    gs = GpuScene(sc)
    params = dict(means=gs.means, scales=gs.scales, quats=gs.quats, opacity=gs.opacity, colors=gs.colors)
    dls = [to_dev(sc.dL_dimage[0])] * 3
    grads = MV.render_views(cams, params, dls)
    torch.cuda.synchronize()
    ref = None
    for cam in cams:
        f = oracle.forward_backward(cam, sc.means, sc.scales, sc.quats, sc.opacity, sc.colors, sc.dL_dimage[0],
                                    "f64")
        ref = {k: f[k] for k in MV.GRAD_KEYS} if ref is None else {k: ref[k] + f[k] for k in MV.GRAD_KEYS}
    for k in MV.GRAD_KEYS:
        assert rel_l2(to_np(grads[k]), ref[k]) <= GRAD_REL_L2, k


def test_render_views_overlapped_equals_sequential():
    """Views whose projection and binning run ahead on the binning stream
    give the gradients of the sequential path (same terms; only the order of
    the floating-point atomics differs), eagerly twice in a row and replayed
    from a CUDA graph."""
    from differentiable_gaussian_splatting_preprocess_b200 import multiview as MV
    sc = _scene(2)
    base = sc.cameras[0]
    cams = [base, base.replace(R=(0.985, 0.0, 0.174, 0.0, 1.0, 0.0, -0.174, 0.0, 0.985)),
            base.replace(t=(0.2, -0.1, 0.0))]
    gs = GpuScene(sc)
    params = dict(means=gs.means, scales=gs.scales, quats=gs.quats, opacity=gs.opacity, colors=gs.colors)
    dls = [to_dev(sc.dL_dimage[0])] * 3
    rzs = {}
    ref = {k: to_np(v).copy() for k, v in MV.render_views(cams, params, dls, rasterizers=rzs).items()
           if k in MV.GRAD_KEYS}
    torch.cuda.synchronize()
    caps = [rzs[i]._bufs["ids"].numel() for i in range(len(cams))]
    for _ in range(2):
        got = MV.render_views(cams, params, dls, rasterizers=rzs, capacity=caps, overlap=True)
        torch.cuda.synchronize()
        for k in MV.GRAD_KEYS:
            assert rel_l2(to_np(got[k]), ref[k]) <= 1e-5, k
    grads = {k: torch.zeros_like(v) for k, v in got.items() if k in MV.GRAD_KEYS}
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture, on a side stream
        MV.render_views(cams, params, dls, grads=grads, rasterizers=rzs, capacity=caps, overlap=True)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for v in grads.values():
            v.zero_()
        MV.render_views(cams, params, dls, grads=grads, rasterizers=rzs, capacity=caps, overlap=True)
    graph.replay()
    torch.cuda.synchronize()
    for k in MV.GRAD_KEYS:
        assert rel_l2(to_np(grads[k]), ref[k]) <= 1e-5, k
    assert all(rz.status() == 0 for rz in rzs.values())


def test_render_views_from_host_overlapped_copies():
    """The host-input step (copies on a side stream, compositing and backward
    waiting on their inputs' events, capacity mode) gives the gradients of the
    device-input path, twice in a row (buffers and stream reused)."""
    from differentiable_gaussian_splatting_preprocess_b200 import multiview as MV
    sc = _scene(2)
    base = sc.cameras[0]
    cams = [base, base.replace(R=(0.985, 0.0, 0.174, 0.0, 1.0, 0.0, -0.174, 0.0, 0.985))]
    gs = GpuScene(sc)
    params = dict(means=gs.means, scales=gs.scales, quats=gs.quats, opacity=gs.opacity, colors=gs.colors)
    dl_np = [sc.dL_dimage[0], -0.5 * sc.dL_dimage[0]]
    ref = MV.render_views(cams, params, [to_dev(d) for d in dl_np])
    torch.cuda.synchronize()
    host = {k: torch.from_numpy(np.ascontiguousarray(getattr(sc, k))).pin_memory()
            for k in ("means", "scales", "quats", "opacity", "colors")}
    host_dl = [torch.from_numpy(np.ascontiguousarray(d)).pin_memory() for d in dl_np]
    out = {k: torch.empty(tuple(ref[k].shape), pin_memory=True) for k in MV.GRAD_KEYS}
    rzs, state = {}, {}
    for _ in range(2):
        MV.render_views_from_host(cams, host, host_dl, rzs, [200_000, 200_000], state=state, host_grads=out)
        torch.cuda.synchronize()
        for k in MV.GRAD_KEYS:
            assert rel_l2(out[k].numpy(), to_np(ref[k])) <= 1e-5, k
    assert all(rz.status() == 0 for rz in rzs.values())
    # pipelined: double-buffered inputs and gradients, copy-back on its own
    # stream, no wait between steps; every step's gradients are the same
    outs = []
    pstate = {}
    for _ in range(4):
        o = {k: torch.empty(tuple(ref[k].shape), pin_memory=True) for k in MV.GRAD_KEYS}
        MV.render_views_from_host(cams, host, host_dl, rzs, [200_000, 200_000], state=pstate, host_grads=o,
                                  pipelined=True)
        outs.append((o, pstate["done"]))
    for o, done in outs:
        done.synchronize()
        for k in MV.GRAD_KEYS:
            assert rel_l2(o[k].numpy(), to_np(ref[k])) <= 1e-5, k


def test_cuda_graph_replay_matches_eager():
    """A whole frame (forward + backward in capacity mode) recorded in a CUDA
    graph and replayed gives the eager results: every call is capturable (no
    host round trip, no attribute or allocation call during capture)."""
    from differentiable_gaussian_splatting_preprocess_b200 import rasterizer as RZ
    sc = _scene(3)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    dl = to_dev(sc.dL_dimage[0])
    rz = RZ.Rasterizer(cam)
    cap = 1_200_000
    grads = RZ.zero_grads(sc.N, gs.means.device)

    def frame():
        for v in grads.values():
            v.zero_()
        fr = rz.forward(gs.means, gs.scales, gs.quats, gs.opacity, gs.colors, capacity=cap)
        rz.backward(fr, gs.means, gs.scales, gs.quats, gs.colors, dl, grads=grads)
        return fr

    fr = frame()
    torch.cuda.synchronize()
    ref = dict(image=to_np(fr.image).copy(), ids=to_np(fr.ids).copy(), ranges=to_np(fr.ranges).copy(),
               **{k: to_np(grads[k]).copy() for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity")})
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fr2 = frame()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert rz.status() == 0
    np.testing.assert_array_equal(to_np(fr2.image), ref["image"])
    np.testing.assert_array_equal(to_np(fr2.ids), ref["ids"])
    np.testing.assert_array_equal(to_np(fr2.ranges), ref["ranges"])
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity"):
        assert rel_l2(to_np(grads[k]), ref[k]) <= 1e-5, k
    del g
    # the same through the library's helper, with inputs updated in place
    # between replays
    gstep = RZ.GraphedStep(RZ.Rasterizer(cam), gs.means, gs.scales, gs.quats, gs.opacity, gs.colors, dl, cap)
    for _ in range(2):
        out = gstep.replay()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(gstep.frame.image), ref["image"])
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity"):
        assert rel_l2(to_np(out[k]), ref[k]) <= 1e-5, k
    gs.colors.mul_(0.5)
    gstep.replay()
    torch.cuda.synchronize()
    assert gstep.status() == 0
    assert not np.array_equal(to_np(gstep.frame.image), ref["image"])
    gs.colors.mul_(2.0)
    # the status word reports the latest replay: larger Gaussians overflow
    # the capacity, the original ones fit again
    orig = gs.scales.clone()
    gs.scales.mul_(3.0)
    gstep.replay()
    assert gstep.status() & B.GS_ERR_CAPACITY
    gs.scales.copy_(orig)
    gstep.replay()
    assert gstep.status() == 0
    np.testing.assert_array_equal(to_np(gstep.frame.image), ref["image"])


def test_image_space_split_equals_full_frame():
    """Tile-aligned bands of one frame (split_image), rendered as separate
    views with their 3D gradients summed, reproduce the full frame: the band
    images are the frame's rows (same bars as the oracle parity), and the
    summed gradients are the frame's."""
    from differentiable_gaussian_splatting_preprocess_b200 import multiview as MV
    from differentiable_gaussian_splatting_preprocess_b200 import rasterizer as RZ
    sc = _scene(3)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    params = dict(means=gs.means, scales=gs.scales, quats=gs.quats, opacity=gs.opacity, colors=gs.colors)
    dl = sc.dL_dimage[0]
    rz = RZ.Rasterizer(cam)
    fr = rz.forward(gs.means, gs.scales, gs.quats, gs.opacity, gs.colors)
    full = rz.backward(fr, gs.means, gs.scales, gs.quats, gs.colors, to_dev(dl))
    torch.cuda.synchronize()
    image, n_contrib = to_np(fr.image), to_np(fr.n_contrib)
    bands, rows = MV.split_image(cam, 3), MV.band_rows(cam, 3)
    rzs = {}
    grads = MV.render_views(bands, params, [to_dev(np.ascontiguousarray(dl[:, y0:y1])) for y0, y1 in rows],
                            rasterizers=rzs)
    torch.cuda.synchronize()
    for i, (y0, y1) in enumerate(rows):
        bf = rzs[i]._bufs
        err = np.abs(to_np(bf["image"]) - image[:, y0:y1])
        assert (err <= IMAGE_ATOL).mean() >= N_CONTRIB_MATCH
        assert (to_np(bf["n_contrib"]) == n_contrib[y0:y1]).mean() >= N_CONTRIB_MATCH
    for k in ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors"):
        assert rel_l2(to_np(grads[k]), to_np(full[k])) <= GRAD_REL_L2, k


def test_autograd_binding_matches_direct_backward():
    """rasterize() under torch.autograd: the image is the forward's, and
    backpropagating sum(image * dL) gives the direct backward's gradients,
    including through user-side activations (scales = exp, opacity = sigmoid)."""
    from differentiable_gaussian_splatting_preprocess_b200 import autograd as AG
    from differentiable_gaussian_splatting_preprocess_b200 import rasterizer as RZ
    sc = _scene(2)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    dl = to_dev(sc.dL_dimage[0])
    rz_ref = RZ.Rasterizer(cam)
    fr = rz_ref.forward(gs.means, gs.scales, gs.quats, gs.opacity, gs.colors)
    ref = rz_ref.backward(fr, gs.means, gs.scales, gs.quats, gs.colors, dl)
    torch.cuda.synchronize()
    log_s = torch.log(gs.scales).requires_grad_(True)
    logit = torch.logit(gs.opacity).requires_grad_(True)
    means = gs.means.clone().requires_grad_(True)
    quats = gs.quats.clone().requires_grad_(True)
    colors = gs.colors.clone().requires_grad_(True)
    rz = RZ.Rasterizer(cam)
    img = AG.rasterize(means, torch.exp(log_s), quats, torch.sigmoid(logit), colors, rz)
    (img * dl).sum().backward()
    torch.cuda.synchronize()
    assert rel_l2(to_np(img.detach()), to_np(fr.image)) <= 1e-6
    for t, k in ((means, "dL_dmeans"), (quats, "dL_dquats"), (colors, "dL_dcolors")):
        assert rel_l2(to_np(t.grad), to_np(ref[k])) <= 1e-5, k
    s = torch.exp(log_s).detach()
    assert rel_l2(to_np(log_s.grad), to_np(ref["dL_dscales"] * s)) <= 1e-5
    o = torch.sigmoid(logit).detach()
    assert rel_l2(to_np(logit.grad), to_np(ref["dL_dopacity"] * o * (1 - o))) <= 1e-5


def test_launch_count_is_fixed_per_frame():
    """The library's launch counter: every frame of one configuration issues
    the same number of kernels (no host-dependent fallbacks), and only the
    library's own launches count."""
    sc = _scene(2)
    cam = sc.cameras[0]
    gs = GpuScene(sc)
    run_gpu(gs, cam, dL_dimage=sc.dL_dimage[0], capacity=200_000)
    deltas = []
    for _ in range(2):
        n0 = B.launch_count()
        run_gpu(gs, cam, dL_dimage=sc.dL_dimage[0], capacity=200_000)
        deltas.append(B.launch_count() - n0)
    assert deltas[0] == deltas[1] > 10
    n0 = B.launch_count()
    torch.zeros(1000, device="cuda").add_(1.0)
    torch.cuda.synchronize()
    assert B.launch_count() == n0
