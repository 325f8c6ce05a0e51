"""gs_preprocess_fwd_noalloc against gs_preprocess_fwd.

The no-allocation entry point serves callers that cannot allocate device
memory themselves (a plug-in whose host application owns every device byte,
or a per-frame loop that must not call cudaMalloc because it synchronises the
device).  Its scratch is a fixed array inside libgs.so, so these tests check
that, called through the C ABI twice in a row, it returns exactly what the
workspace version returns (preprocess outputs are bit-exact by design), and
that a problem above its fixed limit is refused without touching the device.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from differentiable_gaussian_splatting_preprocess_b200 import binding as B
from differentiable_gaussian_splatting_preprocess_b200 import build as BUILD
from differentiable_gaussian_splatting_preprocess_b200 import scenes

pytestmark = pytest.mark.gpu


def _outputs(N, dev):
    f = dict(device=dev)
    return dict(mean2d=torch.empty((N, 2), dtype=torch.float32, **f),
                depth=torch.empty((N,), dtype=torch.float32, **f),
                conic_opacity=torch.empty((N, 4), dtype=torch.float32, **f),
                radius=torch.empty((N,), dtype=torch.int32, **f),
                rect=torch.empty((N, 4), dtype=torch.int32, **f),
                tiles_touched=torch.empty((N,), dtype=torch.uint32, **f),
                num_pairs=torch.empty((1,), dtype=torch.uint32, **f))


def _np(t):
    if t.dtype == torch.uint32:
        return t.view(torch.int32).cpu().numpy().view(np.uint32)
    return t.cpu().numpy()


@pytest.mark.parametrize("cfg", [2, 3])
def test_noalloc_matches_workspace_version_twice(cfg):
    BUILD.build()
    dev = torch.device("cuda", 0)
    sc = scenes.preset(cfg)
    cam = sc.cameras[0]
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    means, scales, quats, opacity = (t(x) for x in (sc.means, sc.scales, sc.quats, sc.opacity))
    N = sc.N

    ref = _outputs(N, dev)
    ws = torch.zeros(B.gs_workspace_bytes(B.GS_STAGE_PREPROCESS_FWD, N, 0, cam.width, cam.height),
                     dtype=torch.uint8, device=dev)
    B.gs_preprocess_fwd(cam, means, scales, quats, opacity, ref["mean2d"], ref["depth"], ref["conic_opacity"],
                        ref["radius"], ref["rect"], ref["tiles_touched"], ref["num_pairs"], ws)
    torch.cuda.synchronize(dev)
    assert B.gs_read_status(ws) == B.GS_OK

    for _ in range(2):
        out = _outputs(N, dev)
        for v in out.values():
            v.view(torch.uint8).fill_(0xAB)  # poison, so stale values cannot pass
        B.gs_preprocess_fwd_noalloc(cam, means, scales, quats, opacity, out["mean2d"], out["depth"],
                                    out["conic_opacity"], out["radius"], out["rect"], out["tiles_touched"],
                                    out["num_pairs"])
        torch.cuda.synchronize(dev)
        for k in ref:
            a, b = _np(out[k]), _np(ref[k])
            if a.dtype.kind == "f":
                a, b = a.view(np.uint32), b.view(np.uint32)
            np.testing.assert_array_equal(a, b, err_msg=k)
        assert int(_np(out["num_pairs"])[0]) == int(_np(ref["tiles_touched"]).astype(np.uint64).sum())


def test_noalloc_refuses_sizes_above_its_limit():
    lib = B.lib()
    fn = lib.gs_preprocess_fwd_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(B.GsCamera), ctypes.c_int] + [ctypes.c_void_p] * 11 + [ctypes.c_void_p]
    cam = B.camera_struct(scenes.Camera(64, 64, 64.0, 64.0, 32.0, 32.0))
    dummy = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    rc = fn(ctypes.byref(cam), B.NOALLOC_MAX_GAUSSIANS + 1, *([dummy] * 11), None)
    assert rc == B.GS_ERR_INVALID_ARG
