"""Host logic of the camera-parallel path, on CPU with two gloo ranks (no GPU):
cameras are split so that each is rendered exactly once, the per-rank sums are
added by one all-reduce, and a rank that fails is noticed by the other
through the process group's timeout instead of a hang."""
import os
import socket
from datetime import timedelta

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from differentiable_gaussian_splatting_preprocess_b200 import multiview as MV


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _row_weight(c, y0, y1):
    """Fake gradient of rows [y0, y1) of camera c: sum of (c + 1)(y + 1)."""
    return float((c + 1) * ((y1 * (y1 + 1) - y0 * (y0 + 1)) // 2))


def _fake_render(cams, params, dls, grads=None, camera_ids=None, **kw):
    """Stands in for the per-view kernels: the unit's rows of camera c add
    _row_weight to every gradient, and the unit is recorded."""
    for view, u in zip(cams, camera_ids):
        assert view.height == u.y1 - u.y0 and view.cy == CAM_H / 2.0 - u.y0
        for k in MV.GRAD_KEYS:
            grads[k] += _row_weight(u.camera, u.y0, u.y1)
        grads["_seen"].append((u.camera, u.y0, u.y1))
    return grads


CAM_H = 1080


def _cams(n_cams, height=CAM_H):
    from differentiable_gaussian_splatting_preprocess_b200 import scenes
    return [scenes.Camera(1920, height, 1600.0, 1600.0, 960.0, CAM_H / 2.0) for _ in range(n_cams)]


def _worker(rank, world, port, n_cams, N, out_q, fail_rank, height=CAM_H):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=10))
    try:
        if rank == fail_rank:
            raise RuntimeError("injected failure before the gradient exchange")
        params = dict(means=torch.zeros(N, 3))
        grads = {k: torch.zeros(s) for k, s in (("dL_dmeans", (N, 3)), ("dL_dscales", (N, 3)),
                                                   ("dL_dquats", (N, 4)), ("dL_dopacity", (N,)),
                                                   ("dL_dcolors", (N, 3)))}
        grads["_seen"] = []
        MV.render_views_distributed(_cams(n_cams, height), params, [None] * n_cams, render_fn=_fake_render,
                                    grads=grads)
        # numpy copies: torch tensors would travel by file-descriptor sharing,
        # which needs this process alive when the parent unpickles them
        out_q.put((rank, "ok", grads["_seen"], {k: grads[k].numpy().copy() for k in MV.GRAD_KEYS}))
    except Exception as e:  # reported to the parent, never swallowed
        out_q.put((rank, "error", type(e).__name__, str(e)[:200]))
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


def _run(world, n_cams, N, fail_rank=-1, height=CAM_H):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n_cams, N, q, fail_rank, height))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    return sorted(res, key=lambda r: r[0])


def test_assign_cameras_partition():
    for world in (1, 2, 3, 4, 8):
        seen = sorted(c for r in range(world) for c in MV.assign_cameras(5, world, r))
        assert seen == list(range(5))
    with pytest.raises(ValueError):
        MV.assign_cameras(4, 2, 2)


def test_flat_roundtrip():
    g = {k: torch.randn(s) for k, s in (("dL_dmeans", (5, 3)), ("dL_dscales", (5, 3)), ("dL_dquats", (5, 4)),
                                         ("dL_dopacity", (5,)), ("dL_dcolors", (5, 3)))}
    flat = MV.flat_grads(g)
    assert flat.numel() == 5 * 14
    h = {k: torch.zeros_like(v) for k, v in g.items()}
    MV.unflatten_into(flat, h)
    for k in g:
        assert torch.equal(g[k], h[k])


@pytest.mark.parametrize("world,n_cams", [(2, 4), (2, 3), (3, 4), (8, 4), (3, 1)])
def test_ranks_render_every_row_once_and_sum(world, n_cams):
    """Every pixel row of every camera is rendered by exactly one rank (whole
    cameras, or bands when the ranks outnumber or do not divide the
    cameras), and after the all-reduce every rank holds the full sum."""
    res = _run(world, n_cams, 7)
    assert all(r[1] == "ok" for r in res), res
    covered = {c: [] for c in range(n_cams)}
    for r in res:
        assert r[2], "every rank has work"
        for c, y0, y1 in r[2]:
            covered[c].append((y0, y1))
    for c, spans in covered.items():
        spans.sort()
        assert spans[0][0] == 0 and spans[-1][1] == CAM_H
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:])), spans
        assert all(y0 % 16 == 0 for y0, _ in spans)
    total = sum(_row_weight(c, 0, CAM_H) for c in range(n_cams))
    for r in res:
        for k, v in r[3].items():
            assert (v == total).all(), k


def test_rank_without_work_contributes_zeros():
    """One tile row and two ranks: the second rank gets no band, renders
    nothing and still joins the all-reduce."""
    res = _run(2, 1, 5, height=16)
    assert all(r[1] == "ok" for r in res), res
    assert res[0][2] == [(0, 0, 16)] and res[1][2] == []
    for r in res:
        for v in r[3].values():
            assert (v == _row_weight(0, 0, 16)).all()


def test_assign_work_partition():
    """The unit assignment alone, for many world sizes: a partition of every
    camera's rows into tile-aligned spans, equal unit counts per rank."""
    for n_cams in (1, 2, 3, 4, 5):
        cams = _cams(n_cams)
        for world in range(1, 17):
            spans = {c: [] for c in range(n_cams)}
            for r in range(world):
                for u in MV.assign_work(cams, world, r):
                    spans[u.camera].append((u.y0, u.y1))
                    assert u.whole == (u.y0 == 0 and u.y1 == CAM_H)
            for c, sp in spans.items():
                sp.sort()
                assert sp[0][0] == 0 and sp[-1][1] == CAM_H and all(a[1] == b[0] for a, b in zip(sp, sp[1:]))
    with pytest.raises(ValueError):
        MV.assign_work(_cams(2), 2, 2)


def test_failed_rank_is_reported_not_hung():
    res = _run(2, 4, 7, fail_rank=1)
    assert res[1][1] == "error" and "injected" in res[1][3]
    # rank 0 reaches the all-reduce alone and gets an error from the timeout
    assert res[0][1] == "error"


def test_split_image_bands_cover_the_frame():
    from differentiable_gaussian_splatting_preprocess_b200 import scenes
    cam = scenes.Camera(1920, 1080, 1600.0, 1600.0, 960.0, 540.0)
    for parts in (1, 2, 3, 8, 68, 100):
        bands = MV.split_image(cam, parts)
        rows = MV.band_rows(cam, parts)
        assert len(bands) == len(rows) <= min(parts, 68)
        assert rows[0][0] == 0 and rows[-1][1] == 1080
        for (a0, a1), (b0, b1) in zip(rows, rows[1:]):
            assert a1 == b0 and a0 % 16 == 0
        for bc, (y0, y1) in zip(bands, rows):
            assert bc.height == y1 - y0 and bc.cy == cam.cy - y0 and bc.width == cam.width
    with pytest.raises(ValueError):
        MV.split_image(cam, 0)
