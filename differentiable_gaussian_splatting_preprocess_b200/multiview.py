"""Several cameras of one scene: render each view forward and backward and sum
the 3D gradients (the views of the 3M-Gaussian scene are rendered back to back
with gradients accumulated).  Across processes the cameras are split between
ranks and the per-rank sums are added with one all-reduce of a single flat
buffer - the only exchange this path has (the Gaussians are replicated; each
view is independent).  On GPUs the process group is NCCL over NVLink; the
host logic is the same for any backend.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Optional, Sequence

import torch
import torch.distributed as dist

from . import rasterizer as RZ

GRAD_KEYS = ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors")


def band_rows(cam, parts: int, tile: int = 16) -> List[tuple]:
    """Pixel row ranges [y0, y1) of ``parts`` horizontal bands of whole tile
    rows (ceil(rows / parts) tile rows each, the last band the remainder;
    empty bands, when the image has fewer tile rows than parts, are omitted)."""
    if parts < 1:
        raise ValueError("parts must be >= 1")
    rows = (cam.height + tile - 1) // tile
    per = (rows + parts - 1) // parts
    out = []
    for b in range(parts):
        r0, r1 = b * per, min(rows, (b + 1) * per)
        if r0 < r1:
            out.append((r0 * tile, min(cam.height, r1 * tile)))
    return out


def split_image(cam, parts: int, tile: int = 16) -> List:
    """Image-space split of one camera into the bands of band_rows.

    A band is the same camera with its principal point moved up by the
    band's first pixel row: every pixel keeps its position relative to the
    Gaussians, and tile rows coincide with the full frame's.  Because the
    preprocess backward is linear in the 2D gradients, the 3D gradients of
    the bands, summed, are those of the full frame: the band renders can run
    on different ranks and meet in the same single all-reduce as the
    camera-parallel split."""
    return [cam.replace(height=y1 - y0, cy=cam.cy - y0) for y0, y1 in band_rows(cam, parts, tile)]


def assign_cameras(n_cameras: int, world: int, rank: int) -> List[int]:
    """Cameras of one rank: round-robin, so every camera belongs to exactly
    one rank and the shares differ by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world size")
    return [i for i in range(n_cameras) if i % world == rank]


def render_views(cams: Sequence, params: Dict[str, torch.Tensor], dL_dimages: Sequence[torch.Tensor],
                 grads: Optional[Dict[str, torch.Tensor]] = None,
                 rasterizers: Optional[Dict[int, "RZ.Rasterizer"]] = None,
                 densify: Optional[Dict[str, torch.Tensor]] = None, capacity: Optional[Sequence[int]] = None,
                 camera_ids: Optional[Sequence[int]] = None) -> Dict[str, torch.Tensor]:
    """Forward and backward of every camera in ``cams``; 3D gradients are
    accumulated into ``grads`` (allocated when None).  ``rasterizers`` caches
    one Rasterizer (and its buffers) per camera id across calls."""
    means, scales, quats = params["means"], params["scales"], params["quats"]
    opacity, colors = params["opacity"], params["colors"]
    if grads is None:
        grads = RZ.zero_grads(means.shape[0], means.device)
    ids = list(range(len(cams))) if camera_ids is None else list(camera_ids)
    for n, (cam, dl) in enumerate(zip(cams, dL_dimages)):
        cid = ids[n]
        rz = None if rasterizers is None else rasterizers.get(cid)
        if rz is None:
            rz = RZ.Rasterizer(cam, means.device)
            if rasterizers is not None:
                rasterizers[cid] = rz
        cap = None if capacity is None else capacity[n]
        fr = rz.forward(means, scales, quats, opacity, colors, capacity=cap)
        rz.backward(fr, means, scales, quats, colors, dl, grads=grads, densify=densify)
    return grads


GEOMETRY_KEYS = ("means", "scales", "quats", "opacity")


def render_views_from_host(cams: Sequence, host_params: Dict[str, torch.Tensor], host_dls: Sequence[torch.Tensor],
                           rasterizers: Dict[int, "RZ.Rasterizer"], capacity: Sequence[int],
                           camera_ids: Optional[Sequence[int]] = None, state: Optional[dict] = None,
                           host_grads: Optional[Dict[str, torch.Tensor]] = None,
                           reduce_fn: Optional[Callable[[Dict[str, torch.Tensor]], None]] = None,
                           device=None, pipelined: bool = False) -> Dict[str, torch.Tensor]:
    """One training step's rasterization from host (pinned) inputs to host
    gradients, with the copies overlapped with the kernels.

    The inputs move to device buffers on a side stream, in the order the
    stages read them: the geometry (means, scales, quats, opacity) first -
    the projection waits for it - then the colours, which the compositing
    waits for while projection and binning run, then each view's dL/dimage,
    which only its backward waits for.  Every view runs in capacity mode
    (``capacity[n]`` pairs, no host round trip).  ``reduce_fn`` (e.g. the
    cross-rank all-reduce) runs on the summed gradients before they are
    copied to ``host_grads``.  ``state`` keeps the streams and buffers across
    steps.

    Without ``pipelined`` the gradients are copied back on the compute stream
    (the caller synchronises it before reading ``host_grads``).  With
    ``pipelined`` the device buffers are double-buffered and the copy back
    runs on a third stream: step k+1's inputs are copied while step k
    computes and step k-1's gradients are copied back, and the call returns
    without waiting; ``state["done"]`` is an event that completes when this
    step's gradients are in ``host_grads``."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    st = state if state is not None else {}
    cur = torch.cuda.current_stream(dev)
    nslot = 2 if pipelined else 1
    if "stream" not in st or st.get("nslot") != nslot:
        st.clear()
        st["nslot"] = nslot
        st["stream"] = torch.cuda.Stream(dev)
        st["d2h"] = torch.cuda.Stream(dev)
        st["params"] = [{k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in host_params.items()}
                        for _ in range(nslot)]
        st["dls"] = [[torch.empty(h.shape, dtype=h.dtype, device=dev) for h in host_dls] for _ in range(nslot)]
        st["grads"] = [RZ.zero_grads(host_params["means"].shape[0], dev) for _ in range(nslot)]
        st["freed"] = [None] * nslot  # per slot: event after which its buffers may be overwritten
        st["slot"] = -1
    slot = st["slot"] = (st["slot"] + 1) % nslot
    cs, dp, dd, grads = st["stream"], st["params"][slot], st["dls"][slot], st["grads"][slot]
    if st["freed"][slot] is not None:
        cs.wait_event(st["freed"][slot])  # the readers of this slot's inputs are done
    else:
        cs.wait_stream(cur)
    with torch.cuda.stream(cs):
        for k in GEOMETRY_KEYS:
            dp[k].copy_(host_params[k], non_blocking=True)
        e_geo = torch.cuda.Event()
        e_geo.record(cs)
        dp["colors"].copy_(host_params["colors"], non_blocking=True)
        e_col = torch.cuda.Event()
        e_col.record(cs)
        e_dl = []
        for d, h in zip(dd, host_dls):
            d.copy_(h, non_blocking=True)
            e = torch.cuda.Event()
            e.record(cs)
            e_dl.append(e)
    d2h_prev = st.get("d2h_done", [None] * nslot)[slot]
    if d2h_prev is not None:
        cur.wait_event(d2h_prev)  # this slot's gradients of two steps ago are back on the host
    cur.wait_event(e_geo)
    for v in grads.values():
        v.zero_()
    ids = list(range(len(cams))) if camera_ids is None else list(camera_ids)
    for n, cam in enumerate(cams):
        rz = rasterizers.get(ids[n])
        if rz is None:
            rz = rasterizers[ids[n]] = RZ.Rasterizer(cam, dev)
        fr = rz.forward(dp["means"], dp["scales"], dp["quats"], dp["opacity"], dp["colors"], capacity=capacity[n],
                        colors_ready=e_col)
        rz.backward(fr, dp["means"], dp["scales"], dp["quats"], dp["colors"], dd[n], grads=grads,
                    dL_ready=e_dl[n])
    if reduce_fn is not None:
        reduce_fn(grads)
    computed = torch.cuda.Event()
    computed.record(cur)
    st["freed"][slot] = computed
    if host_grads is not None:
        if pipelined:
            ds = st["d2h"]
            ds.wait_event(computed)
            with torch.cuda.stream(ds):
                for k, h in host_grads.items():
                    h.copy_(grads[k], non_blocking=True)
            done = torch.cuda.Event()
            done.record(ds)
            st.setdefault("d2h_done", [None] * nslot)[slot] = done
            st["done"] = done
        else:
            for k, h in host_grads.items():
                h.copy_(grads[k], non_blocking=True)
            done = torch.cuda.Event()
            done.record(cur)
            st["done"] = done
    return grads


def flat_grads(grads: Dict[str, torch.Tensor], keys: Sequence[str] = GRAD_KEYS) -> torch.Tensor:
    return torch.cat([grads[k].reshape(-1) for k in keys])


def unflatten_into(flat: torch.Tensor, grads: Dict[str, torch.Tensor], keys: Sequence[str] = GRAD_KEYS) -> None:
    off = 0
    for k in keys:
        n = grads[k].numel()
        grads[k].copy_(flat[off:off + n].view_as(grads[k]))
        off += n


def allreduce_grads(grads: Dict[str, torch.Tensor], group=None, keys: Sequence[str] = GRAD_KEYS) -> None:
    """Sum the gradient tensors over the ranks of ``group`` in place, with one
    all-reduce of a single contiguous buffer (one launch, one NVLink
    transfer schedule, whatever the number of tensors)."""
    flat = flat_grads(grads, keys)
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    unflatten_into(flat, grads, keys)


def render_views_distributed(cams: Sequence, params: Dict[str, torch.Tensor],
                             dL_dimages: Sequence[torch.Tensor], group=None,
                             render_fn: Callable = render_views, **kw) -> Dict[str, torch.Tensor]:
    """Each rank renders its share of the cameras (assign_cameras), then the
    3D gradients are summed over ranks: every rank ends with the gradient of
    the sum of all views' losses."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    mine = assign_cameras(len(cams), world, rank)
    grads = kw.pop("grads", None)
    if grads is None:
        grads = RZ.zero_grads(params["means"].shape[0], params["means"].device)
    render_fn([cams[i] for i in mine], params, [dL_dimages[i] for i in mine], grads=grads, camera_ids=mine, **kw)
    if world > 1:
        allreduce_grads(grads, group)
    return grads
