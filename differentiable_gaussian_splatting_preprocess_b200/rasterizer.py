"""A frame-level driver over the C ABI: allocates device buffers with torch,
calls the five stages in order on the current stream, and keeps the forward's
buffers (sorted ids, tile ranges, final transmittance, contributor counts) for
the backward, as the backward of "Gaussian Splatting反向传播的CUDA实现"
(section 1) reuses them.  All arithmetic runs in libgs.so.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

from . import binding as B


@dataclasses.dataclass
class Frame:
    """Buffers of one forward pass (device tensors)."""
    N: int
    capacity: int
    mean2d: torch.Tensor
    depth: torch.Tensor
    conic_opacity: torch.Tensor
    radius: torch.Tensor
    rect: torch.Tensor
    tiles_touched: torch.Tensor
    num_pairs: torch.Tensor      # [1] uint32, on the device
    ids: torch.Tensor
    ranges: torch.Tensor
    keys: Optional[torch.Tensor]
    image: torch.Tensor
    final_T: torch.Tensor
    n_contrib: torch.Tensor
    contrib_mask: Optional[torch.Tensor]


class Rasterizer:
    """One camera's rasterizer with cached device buffers.

    Buffers are reused across calls while N, the capacity and the image size
    stay the same, so repeated frames allocate nothing.  The workspace is
    zero-filled when it is (re)allocated, as the C ABI requires.
    """

    def __init__(self, cam, device: Optional[torch.device] = None):
        self.cam = cam
        self.device = torch.device("cuda") if device is None else torch.device(device)
        self._bufs: Dict[str, torch.Tensor] = {}
        self.ws: Optional[torch.Tensor] = None

    # -- buffers ----------------------------------------------------------
    def _buf(self, name: str, shape, dtype, zero: bool = False) -> torch.Tensor:
        t = self._bufs.get(name)
        if t is None or tuple(t.shape) != tuple(shape) or t.dtype != dtype:
            t = (torch.zeros if zero else torch.empty)(tuple(shape), dtype=dtype, device=self.device)
            self._bufs[name] = t
        return t

    def workspace(self, N: int, capacity: int) -> torch.Tensor:
        W, H = self.cam.width, self.cam.height
        need = max(B.gs_workspace_bytes(B.GS_STAGE_PREPROCESS_FWD, N, 0, W, H),
                   B.gs_workspace_bytes(B.GS_STAGE_BIN_SORT, N, capacity, W, H))
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.zeros(need + (need >> 4), dtype=torch.uint8, device=self.device)
        return self.ws

    # -- stages -----------------------------------------------------------
    def preprocess(self, means, scales, quats, opacity, stream=None):
        N = means.shape[0]
        ws = self.workspace(N, 0)
        out = dict(mean2d=self._buf("mean2d", (N, 2), torch.float32),
                   depth=self._buf("depth", (N,), torch.float32),
                   conic_opacity=self._buf("conic_opacity", (N, 4), torch.float32),
                   radius=self._buf("radius", (N,), torch.int32),
                   rect=self._buf("rect", (N, 4), torch.int32),
                   tiles_touched=self._buf("tiles_touched", (N,), torch.uint32),
                   num_pairs=self._buf("num_pairs", (1,), torch.uint32))
        B.gs_preprocess_fwd(self.cam, means, scales, quats, opacity, out["mean2d"], out["depth"],
                            out["conic_opacity"], out["radius"], out["rect"], out["tiles_touched"],
                            out["num_pairs"], ws, stream)
        return out

    def forward(self, means, scales, quats, opacity, colors, capacity: Optional[int] = None,
                want_keys: bool = False, use_mask: bool = True, stream=None,
                colors_ready: Optional[torch.cuda.Event] = None, render_stream=None) -> Frame:
        """Preprocess, bin/sort and composite one frame.

        With ``capacity=None`` the pair count is read back to size the sort
        buffers (one device-to-host copy).  With a capacity the call makes no
        host round trip; if the frame needs more pairs, the status word of
        the workspace reports GS_ERR_CAPACITY and every tile range is empty.
        ``colors_ready``: an event the compositing waits for (the colours may
        still be arriving while the projection and the binning run).
        ``render_stream``: run the compositing there instead of on
        ``stream``, after the binning (an event joins the two), so that the
        projection and binning of the next frame can go ahead on ``stream``.
        """
        N = means.shape[0]
        pre = self.preprocess(means, scales, quats, opacity, stream)
        if capacity is None:
            with torch.cuda.stream(stream):  # the read waits for the projection
                capacity = int(pre["num_pairs"].to("cpu").view(torch.int32).item()) & 0xFFFFFFFF
        ws = self.workspace(N, capacity)
        ids = self._buf("ids", (max(capacity, 1),), torch.uint32)
        ranges = self._buf("ranges", (B.num_tiles(self.cam), 2), torch.uint32)
        keys = self._buf("keys", (max(capacity, 1),), torch.uint64) if want_keys else None
        B.gs_bin_sort(self.cam, pre["depth"], pre["rect"], pre["tiles_touched"], pre["num_pairs"], capacity, ids,
                      ranges, keys, ws, stream)
        H, W = self.cam.height, self.cam.width
        image = self._buf("image", (3, H, W), torch.float32)
        final_T = self._buf("final_T", (H, W), torch.float32)
        n_contrib = self._buf("n_contrib", (H, W), torch.uint32)
        cmask = (self._buf("contrib_mask", (B.mask_words(max(capacity, 1), B.num_tiles(self.cam)),), torch.uint32)
                 if use_mask else None)
        if render_stream is not None:
            binned = torch.cuda.Event()
            binned.record(stream or torch.cuda.current_stream(self.device))
            render_stream.wait_event(binned)
            stream = render_stream
        if colors_ready is not None:
            (stream or torch.cuda.current_stream(self.device)).wait_event(colors_ready)
        B.gs_render_fwd(self.cam, ranges, ids, pre["mean2d"], pre["conic_opacity"], colors, image, final_T,
                        n_contrib, cmask, stream)
        return Frame(N=N, capacity=capacity, ids=ids, ranges=ranges, keys=keys, image=image, final_T=final_T,
                     n_contrib=n_contrib, contrib_mask=cmask, **pre)

    def backward(self, frame: Frame, means, scales, quats, colors, dL_dimage,
                 grads: Optional[Dict[str, torch.Tensor]] = None, densify: Optional[Dict[str, torch.Tensor]] = None,
                 stream=None, dL_ready: Optional[torch.cuda.Event] = None) -> Dict[str, torch.Tensor]:
        """Render backward then preprocess backward.  3D gradients are
        accumulated into ``grads`` (zeros are allocated when it is None).
        With ``densify`` = dict(grad2d_accum=[N] float32, vis_count=[N] uint32),
        the densification statistics of this view are accumulated too.
        ``dL_ready``: an event the backward waits for before reading
        ``dL_dimage``."""
        N = frame.N
        if dL_ready is not None:
            (stream or torch.cuda.current_stream(self.device)).wait_event(dL_ready)
        g2 = dict(dL_dmean2d=self._buf("dL_dmean2d", (N, 2), torch.float32),
                  dL_dconic_opacity=self._buf("dL_dconic_opacity", (N, 4), torch.float32),
                  dL_dcolor=self._buf("dL_dcolor", (N, 3), torch.float32))
        B.gs_render_bwd(self.cam, frame.ranges, frame.ids, frame.mean2d, frame.conic_opacity, colors, frame.final_T,
                        frame.n_contrib, dL_dimage, g2["dL_dmean2d"], g2["dL_dconic_opacity"], g2["dL_dcolor"],
                        frame.contrib_mask, stream)
        if grads is None:
            grads = zero_grads(N, self.device)
        B.gs_preprocess_bwd(self.cam, means, scales, quats, frame.radius, frame.conic_opacity, g2["dL_dmean2d"],
                            g2["dL_dconic_opacity"], g2["dL_dcolor"], grads["dL_dmeans"], grads["dL_dscales"],
                            grads["dL_dquats"], grads["dL_dopacity"], grads["dL_dcolors"],
                            None if densify is None else densify["grad2d_accum"],
                            None if densify is None else densify["vis_count"], stream)
        grads.update(g2)
        return grads

    def status(self, stream=None) -> int:
        return 0 if self.ws is None else B.gs_read_status(self.ws, stream)


def zero_grads(N: int, device) -> Dict[str, torch.Tensor]:
    f = dict(dtype=torch.float32, device=device)
    return dict(dL_dmeans=torch.zeros((N, 3), **f), dL_dscales=torch.zeros((N, 3), **f),
                dL_dquats=torch.zeros((N, 4), **f), dL_dopacity=torch.zeros((N,), **f),
                dL_dcolors=torch.zeros((N, 3), **f))


class GraphedStep:
    """Forward + backward of one camera recorded once into a CUDA graph and
    replayed: one launch per step instead of one per kernel.

    The inputs are the tensors given here, read in place at every replay
    (update them with ``copy_`` between replays); the step runs in capacity
    mode, so the pair count of every replayed frame must fit ``capacity``.
    ``grads`` (allocated when None) is zeroed and refilled by every replay;
    ``frame`` holds the forward's outputs.

    The graph records device addresses, so the step owns the buffers they
    belong to: it builds its own Rasterizer (from ``cam``, or from the
    camera of a Rasterizer passed instead), whose workspace, pair buffers,
    frame and 2D gradient buffers live as long as the step and are used by
    nothing else.  A Rasterizer passed in is not used and stays free for
    eager calls.  Each replay begins by clearing the workspace's status
    word, so ``status()`` reports the most recent replay (GS_ERR_CAPACITY
    when its pair count did not fit)."""

    def __init__(self, cam, means, scales, quats, opacity, colors, dL_dimage, capacity: int,
                 grads: Optional[Dict[str, torch.Tensor]] = None, use_mask: bool = True):
        if isinstance(cam, Rasterizer):
            cam, device = cam.cam, cam.device
        else:
            device = means.device
        rz = self.rz = Rasterizer(cam, device)
        self.grads = zero_grads(means.shape[0], device) if grads is None else grads
        args = (means, scales, quats, opacity, colors)

        def step():
            if rz.ws is not None:
                B.gs_clear_status(rz.ws)
            for v in self.grads.values():
                v.zero_()
            fr = rz.forward(*args, capacity=capacity, use_mask=use_mask)
            rz.backward(fr, means, scales, quats, colors, dL_dimage, grads=self.grads)
            return fr

        step()  # allocates every buffer and makes every one-time setup call outside the capture
        torch.cuda.synchronize(device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.frame = step()
        # the tensors whose addresses the graph holds
        self.ws = rz.ws
        self._held = (rz.ws, dict(rz._bufs), args, dL_dimage, self.grads)

    def replay(self) -> Dict[str, torch.Tensor]:
        self.graph.replay()
        return self.grads

    def status(self) -> int:
        """Status word of the workspace the graph uses (synchronises)."""
        return B.gs_read_status(self.ws)
