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


def _fake_render(cams, params, dls, grads=None, camera_ids=None, **kw):
    """Stands in for the per-camera kernels: camera c adds (c + 1) * ones to
    every gradient and records that it ran."""
    for cid in camera_ids:
        for k in MV.GRAD_KEYS:
            grads[k] += float(cid + 1)
        grads["_seen"].append(cid)
    return grads


def _worker(rank, world, port, n_cams, N, out_q, fail_rank):
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
        MV.render_views_distributed(list(range(n_cams)), params, [None] * n_cams, render_fn=_fake_render,
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


def _run(world, n_cams, N, fail_rank=-1):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n_cams, N, q, fail_rank)) for r in range(world)]
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


@pytest.mark.parametrize("n_cams", [4, 3])
def test_two_ranks_sum_every_camera_once(n_cams):
    res = _run(2, n_cams, 7)
    assert all(r[1] == "ok" for r in res), res
    seen = sorted(c for r in res for c in r[2])
    assert seen == list(range(n_cams))
    total = float(sum(c + 1 for c in range(n_cams)))
    for r in res:
        for k, v in r[3].items():
            assert (v == total).all(), k


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
