"""torch.autograd binding of the rasterizer: ``rasterize(...)`` returns the
image [3, H, W] of one camera and, when the graph is back-propagated, the
gradients w.r.t. means, scales, quats, opacity and colours (the activated
values the rasterizer consumes).  All work runs in libgs.so through a
``Rasterizer``; this module only connects it to autograd.

The Rasterizer keeps the forward's buffers (sorted ids, tile ranges, final
transmittance, contributor counts, contribution mask) for the backward, so a
Rasterizer must not run another forward before the backward of its previous
one: use one Rasterizer per camera (as ``multiview`` does) when several views
are rendered before one backward.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import rasterizer as RZ


class _Rasterize(torch.autograd.Function):
    @staticmethod
    def forward(ctx, means, scales, quats, opacity, colors, rz: "RZ.Rasterizer", capacity: Optional[int]):
        means, scales, quats = means.contiguous(), scales.contiguous(), quats.contiguous()
        opacity, colors = opacity.contiguous(), colors.contiguous()
        frame = rz.forward(means, scales, quats, opacity, colors, capacity=capacity)
        ctx.rz, ctx.frame = rz, frame
        ctx.save_for_backward(means, scales, quats, colors)
        return frame.image.clone()  # the Rasterizer reuses its image buffer next frame

    @staticmethod
    def backward(ctx, dL_dimage):
        means, scales, quats, colors = ctx.saved_tensors
        g = ctx.rz.backward(ctx.frame, means, scales, quats, colors, dL_dimage.contiguous())
        return g["dL_dmeans"], g["dL_dscales"], g["dL_dquats"], g["dL_dopacity"], g["dL_dcolors"], None, None


def rasterize(means: torch.Tensor, scales: torch.Tensor, quats: torch.Tensor, opacity: torch.Tensor,
              colors: torch.Tensor, rasterizer: "RZ.Rasterizer", capacity: Optional[int] = None) -> torch.Tensor:
    """Image [3, H, W] (float32, channel-major) of ``rasterizer``'s camera.
    Differentiable w.r.t. the five parameter tensors.  ``capacity``: pair
    bound for capacity mode (no host round trip); None sizes it from the
    frame's pair count."""
    return _Rasterize.apply(means, scales, quats, opacity, colors, rasterizer, capacity)
