"""B200-native tile rasterizer for differentiable 3D Gaussian Splatting.

The compute lives in ``libgs.so`` (CUDA kernels for sm_100a behind the C ABI
of ``include/gs.h``); ``binding`` marshals torch tensors to it and
``rasterizer`` drives the five stages for one camera.  ``scenes`` draws seeded
synthetic inputs.
"""
from . import scenes  # noqa: F401

__all__ = ["scenes", "binding", "rasterizer", "build"]
