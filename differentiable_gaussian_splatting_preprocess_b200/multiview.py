"""Several cameras of one scene: render each view forward and backward and sum
the 3D gradients (the views of the 3M-Gaussian scene are rendered back to back
with gradients accumulated).  Across processes the cameras are split between
ranks and the per-rank sums are added with one all-reduce of a single flat
buffer - the only exchange this path has (the Gaussians are replicated; each
view is independent).  On GPUs the process group is NCCL over NVLink; the
host logic is the same for any backend.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, Dict, List, Optional, Sequence

import torch
import torch.distributed as dist

from . import rasterizer as RZ

GRAD_KEYS = ("dL_dmeans", "dL_dscales", "dL_dquats", "dL_dopacity", "dL_dcolors")


def _band_bounds(tile_rows: int, parts: int) -> List[int]:
    """parts + 1 tile-row boundaries: band k holds tile rows
    [ceil(k rows / parts), ceil((k + 1) rows / parts)), so band sizes differ
    by at most one tile row (when rows < parts, the last bands are empty)."""
    if parts < 1:
        raise ValueError("parts must be >= 1")
    return [(k * tile_rows + parts - 1) // parts for k in range(parts + 1)]


def band_rows(cam, parts: int, tile: int = 16) -> List[tuple]:
    """Pixel row ranges [y0, y1) of ``parts`` horizontal bands of whole tile
    rows, as equal as whole tile rows allow; empty bands (when the image has
    fewer tile rows than parts) are omitted."""
    rows = (cam.height + tile - 1) // tile
    b = _band_bounds(rows, parts)
    return [(b[k] * tile, min(cam.height, b[k + 1] * tile)) for k in range(parts) if b[k] < b[k + 1]]


def band_view(cam, y0: int, y1: int):
    """The camera restricted to pixel rows [y0, y1): same camera with its
    principal point moved up by y0, so every pixel keeps its position
    relative to the Gaussians.  y0 must be a multiple of the tile size, so
    that the band's tile rows coincide with the full frame's."""
    return cam.replace(height=y1 - y0, cy=cam.cy - y0)


def split_image(cam, parts: int, tile: int = 16) -> List:
    """Image-space split of one camera into the bands of band_rows.

    The preprocess backward is linear in the 2D gradients, so the 3D
    gradients of the bands, summed, equal those of the full frame up to fp32
    rounding (each band projects the means with its own principal point, so
    the pixel offsets round differently): the band renders can run on
    different ranks and meet in the same single all-reduce as the
    camera-parallel split.  The densification statistics are not linear in
    the 2D gradients (a norm per view), so they must not be summed over
    bands: compute them from whole views only."""
    return [band_view(cam, y0, y1) for y0, y1 in band_rows(cam, parts, tile)]


def assign_cameras(n_cameras: int, world: int, rank: int) -> List[int]:
    """Cameras of one rank: round-robin, so every camera belongs to exactly
    one rank and the shares differ by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world size")
    return [i for i in range(n_cameras) if i % world == rank]


@dataclasses.dataclass(frozen=True)
class WorkUnit:
    """Rows [y0, y1) of camera ``camera``: one rank's share of a step."""
    camera: int
    y0: int
    y1: int
    whole: bool  # the unit is the camera's whole frame


def assign_work(cams: Sequence, world: int, rank: int, tile: int = 16) -> List[WorkUnit]:
    """The (camera, band) work units of one rank, for any number of ranks.

    Each camera is cut into b = world / gcd(n_cameras, world) bands of whole
    tile rows (_band_bounds), which makes n_cameras * b units, a multiple of
    the number of ranks; rank r takes the contiguous run of U = n_cameras * b
    / world units starting at r U, and neighbouring bands of one camera in
    that run are merged into one taller band.  So every pixel row of every
    camera belongs to exactly one rank, every rank gets the same number of
    units, a rank splits a camera only where the ranks outnumber or do not
    divide the cameras, and with world dividing n_cameras it is whole cameras
    per rank.  Empty bands (fewer tile rows than bands) are dropped, so a
    rank of a small image may get no unit: it then contributes zeros to the
    gradient sum."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world size")
    n = len(cams)
    if n == 0:
        return []
    b = world // math.gcd(n, world)
    per = n * b // world
    first, last = rank * per, (rank + 1) * per  # unit u = camera u // b, band u % b
    out = []
    u = first
    while u < last:
        c, k0 = divmod(u, b)
        k1 = min(b, k0 + (last - u))  # bands k0 .. k1 - 1 of camera c
        rows = (cams[c].height + tile - 1) // tile
        bd = _band_bounds(rows, b)
        y0, y1 = bd[k0] * tile, min(cams[c].height, bd[k1] * tile)
        if y0 < y1:
            out.append(WorkUnit(c, y0, y1, y0 == 0 and y1 == cams[c].height))
        u += k1 - k0
    return out


def unit_view(cams: Sequence, unit: WorkUnit):
    """The camera a work unit renders (its band of the unit's camera)."""
    cam = cams[unit.camera]
    return cam if unit.whole else band_view(cam, unit.y0, unit.y1)


_BIN_STREAMS: Dict[int, torch.cuda.Stream] = {}


def binning_stream(device) -> torch.cuda.Stream:
    """The high-priority stream that projects and bins the views ahead of
    their compositing (one per device)."""
    idx = torch.device(device).index
    idx = torch.cuda.current_device() if idx is None else idx
    if idx not in _BIN_STREAMS:
        _BIN_STREAMS[idx] = torch.cuda.Stream(torch.device("cuda", idx), priority=-1)
    return _BIN_STREAMS[idx]


def render_views(cams: Sequence, params: Dict[str, torch.Tensor], dL_dimages: Sequence[torch.Tensor],
                 grads: Optional[Dict[str, torch.Tensor]] = None,
                 rasterizers: Optional[Dict[int, "RZ.Rasterizer"]] = None,
                 densify: Optional[Dict[str, torch.Tensor]] = None, capacity: Optional[Sequence[int]] = None,
                 camera_ids: Optional[Sequence[int]] = None, overlap: bool = False) -> Dict[str, torch.Tensor]:
    """Forward and backward of every camera in ``cams``; 3D gradients are
    accumulated into ``grads`` (allocated when None).  ``rasterizers`` caches
    one Rasterizer (and its buffers) per camera id across calls.

    With ``overlap`` (capacity mode: ``capacity`` given) the views' projection
    and binning run back to back on a high-priority side stream
    (``binning_stream``) while the current stream composites, differentiates
    and accumulates the views in order, each after its own binning: the
    binning of view n + 1, bound by latency, fills the GPU beside the
    compositing of view n.  The views must not share per-view buffers (one
    Rasterizer per camera id), and the colours must not depend on the view."""
    means, scales, quats = params["means"], params["scales"], params["quats"]
    opacity, colors = params["opacity"], params["colors"]
    if grads is None:
        grads = RZ.zero_grads(means.shape[0], means.device)
    ids = list(range(len(cams))) if camera_ids is None else list(camera_ids)
    if overlap and capacity is None:
        raise ValueError("overlapped views run in capacity mode: pass capacity")
    cur = torch.cuda.current_stream(means.device)
    bs = binning_stream(means.device) if overlap else None
    if bs is not None:
        bs.wait_stream(cur)  # inputs written, earlier readers of the per-view buffers done
    for n, (cam, dl) in enumerate(zip(cams, dL_dimages)):
        cid = ids[n]
        rz = None if rasterizers is None else rasterizers.get(cid)
        if rz is None:
            rz = RZ.Rasterizer(cam, means.device)
            if rasterizers is not None:
                rasterizers[cid] = rz
        cap = None if capacity is None else capacity[n]
        fr = rz.forward(means, scales, quats, opacity, colors, capacity=cap, stream=bs,
                        render_stream=cur if bs is not None else None)
        rz.backward(fr, means, scales, quats, colors, dl, grads=grads, densify=densify)
    if bs is not None:
        cur.wait_stream(bs)
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
    """Each rank renders its work units (assign_work: whole cameras, or bands
    of cameras when the ranks outnumber or do not divide the cameras), then
    the 3D gradients are summed over ranks: every rank ends with the gradient
    of the sum of all views' losses.  A rank without a unit contributes
    zeros.  ``render_fn`` receives the units' cameras, their rows of the
    upstream gradients and ``camera_ids`` = the units (hashable keys for a
    rasterizer cache)."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    units = assign_work(cams, world, rank)
    if kw.get("densify") is not None and not all(u.whole for u in units):
        raise ValueError("densification statistics are not additive over image bands")
    grads = kw.pop("grads", None)
    if grads is None:
        grads = RZ.zero_grads(params["means"].shape[0], params["means"].device)
    if units:
        views = [unit_view(cams, u) for u in units]
        dls = [dL_dimages[u.camera] if (u.whole or dL_dimages[u.camera] is None)
               else dL_dimages[u.camera][:, u.y0:u.y1].contiguous() for u in units]
        render_fn(views, params, dls, grads=grads, camera_ids=units, **kw)
    if world > 1:
        allreduce_grads(grads, group)
    return grads
