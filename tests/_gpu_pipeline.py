"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
the oracle on the same seeded inputs, and the comparison metrics."""
from __future__ import annotations

import numpy as np
import torch

from differentiable_gaussian_splatting_preprocess_b200 import rasterizer as RZ

# Tolerances (the acceptance bar): image absolute error, contributor-count
# agreement, per-tensor gradient relative L2 error, all in fp32.
IMAGE_ATOL = 1e-4
N_CONTRIB_MATCH = 0.9999
GRAD_REL_L2 = 1e-3


def to_dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=dtype)


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.uint32:
        return t.view(torch.int32).cpu().numpy().view(np.uint32)
    if t.dtype == torch.uint64:
        return t.view(torch.int64).cpu().numpy().view(np.uint64)
    return t.cpu().numpy()


def rel_l2(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)


class GpuScene:
    """Scene parameters resident on the device."""

    def __init__(self, sc):
        self.sc = sc
        self.means = to_dev(sc.means)
        self.scales = to_dev(sc.scales)
        self.quats = to_dev(sc.quats)
        self.opacity = to_dev(sc.opacity)
        self.colors = to_dev(sc.colors)


def run_gpu(gs: GpuScene, cam, dL_dimage=None, want_keys=True, capacity=None, grads=None):
    rz = RZ.Rasterizer(cam)
    fr = rz.forward(gs.means, gs.scales, gs.quats, gs.opacity, gs.colors, capacity=capacity, want_keys=want_keys)
    out = dict(rz=rz, frame=fr)
    if dL_dimage is not None:
        g = rz.backward(fr, gs.means, gs.scales, gs.quats, gs.colors, to_dev(dL_dimage), grads=grads)
        out["grads"] = g
    torch.cuda.synchronize()
    return out


def frame_np(fr) -> dict:
    P = int(to_np(fr.num_pairs)[0])
    d = dict(mean2d=to_np(fr.mean2d), depth=to_np(fr.depth), conic_opacity=to_np(fr.conic_opacity),
             radius=to_np(fr.radius), rect=to_np(fr.rect), tiles_touched=to_np(fr.tiles_touched), num_pairs=P,
             ranges=to_np(fr.ranges), image=to_np(fr.image), final_T=to_np(fr.final_T),
             n_contrib=to_np(fr.n_contrib))
    d["ids"] = to_np(fr.ids)[:P]
    if fr.keys is not None:
        d["keys"] = to_np(fr.keys)[:P]
    return d
