"""Child process of test_debug_build (run with GS_LIBRARY=debug): drives the
index-checking build of the library and prints one JSON line."""
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from differentiable_gaussian_splatting_preprocess_b200 import binding as B  # noqa: E402
from differentiable_gaussian_splatting_preprocess_b200 import rasterizer as RZ  # noqa: E402
from differentiable_gaussian_splatting_preprocess_b200 import scenes  # noqa: E402


def main():
    assert B.LIB_PATH.endswith("libgs_debug.so"), B.LIB_PATH
    dev = torch.device("cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    out = {"library": os.path.basename(B.LIB_PATH)}
    for cfg in (1, 2, 3, 4):
        sc = scenes.preset(cfg)
        cam = sc.cameras[0]
        means, scales, quats, opacity, colors = (t(x) for x in (sc.means, sc.scales, sc.quats, sc.opacity,
                                                                  sc.colors))
        rz = RZ.Rasterizer(cam, dev)
        B.gs_debug_configure(sc.N, 0xFFFFFFFF)
        fr = rz.forward(means, scales, quats, opacity, colors)  # sizes the pair buffers
        cap = fr.capacity
        # valid run: the real limits
        B.gs_debug_configure(sc.N, cap)
        fr = rz.forward(means, scales, quats, opacity, colors, capacity=cap)
        rz.backward(fr, means, scales, quats, colors, t(sc.dL_dimage[0]))
        clean = B.gs_debug_read(clear=True)
        status = rz.status()
        u32 = lambda x: x.view(torch.int32).cpu().numpy().view(np.uint32)
        o = oracle.render_fwd(cam, u32(fr.ranges), u32(fr.ids)[:int(u32(fr.num_pairs)[0])], fr.mean2d.cpu().numpy(),
                              fr.conic_opacity.cpu().numpy(), sc.colors, "f32")
        same = bool(np.array_equal(u32(fr.n_contrib), o["n_contrib"])
                    and np.abs(fr.image.cpu().numpy() - o["image"]).max() <= 1e-4)
        # limits tighter than the real buffers: the checks fire (every access
        # they stop would still have been inside the real buffers)
        B.gs_debug_configure(sc.N // 2, cap // 2)
        fr = rz.forward(means, scales, quats, opacity, colors, capacity=cap)
        rz.backward(fr, means, scales, quats, colors, t(sc.dL_dimage[0]))
        tight = B.gs_debug_read(clear=True)
        B.gs_debug_configure(sc.N, cap)
        fr = rz.forward(means, scales, quats, opacity, colors, capacity=cap)
        again = B.gs_debug_read(clear=True)
        out[f"config{cfg}"] = dict(clean=clean, status=status, matches_oracle=same, tight=tight, again=again)
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
