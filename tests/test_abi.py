"""The C-ABI library loads and exports every symbol include/gs.h declares, and
its host-side helpers behave; no compute call is made (runs without a GPU)."""
import ctypes
import os
import re

import pytest

from differentiable_gaussian_splatting_preprocess_b200 import binding as B
from differentiable_gaussian_splatting_preprocess_b200 import build as BUILD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.lib()


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"GS_API\s+[\w\s\*]+?\b(gs_\w+)\s*\(", txt))
    return names


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert declared == set(B.EXPORTED)
    for name in declared:
        assert hasattr(lib, name), name


def _prototypes():
    """name -> number of parameters, from the GS_API declarations of include/*.h."""
    protos = {}
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            for name, params in re.findall(r"GS_API\s+[\w\s\*]+?\b(gs_\w+)\s*\(([^)]*)\)", txt):
                params = params.strip()
                protos[name] = 0 if params in ("", "void") else params.count(",") + 1
    return protos


def test_binding_signatures_match_header(lib):
    """Every ctypes prototype of the binding has as many parameters as the C
    declaration, so a call can never be marshalled against the wrong layout."""
    protos = _prototypes()
    assert set(protos) == set(B.EXPORTED)
    for name, n in protos.items():
        assert len(getattr(lib, name).argtypes) == n, name


def test_adam_config_layout_matches_header():
    # float lr x5, beta1, beta2, eps; int warmup_steps
    assert ctypes.sizeof(B.GsAdamConfig) == 4 * 9


def test_camera_struct_layout_matches_header():
    # int width, height, tile; float fx, fy, cx, cy, R[9], t[3], 6 scalars, bg[3]
    assert ctypes.sizeof(B.GsCamera) == 4 * (3 + 4 + 9 + 3 + 6 + 3)


def test_version_and_status_strings(lib):
    assert B.version() >> 16 == 1
    assert B.status_string(B.GS_OK) == "ok"
    assert "capacity" in B.status_string(B.GS_ERR_CAPACITY)
    assert "several" in B.status_string(B.GS_ERR_CAPACITY | B.GS_ERR_TIMEOUT)


def test_workspace_sizes(lib):
    a = B.gs_workspace_bytes(B.GS_STAGE_PREPROCESS_FWD, 1000, 0, 64, 64)
    b = B.gs_workspace_bytes(B.GS_STAGE_PREPROCESS_FWD, 100000, 0, 64, 64)
    assert 256 < a < b
    c = B.gs_workspace_bytes(B.GS_STAGE_BIN_SORT, 1000, 10000, 64, 64)
    d = B.gs_workspace_bytes(B.GS_STAGE_BIN_SORT, 1000, 20000, 64, 64)
    assert d - c >= 4 * 4 * 10000 - 4 * 256  # four pair-sized buffers, each 256-byte aligned
    assert B.gs_workspace_bytes(7, 10, 10, 64, 64) == 0
    assert B.gs_workspace_bytes(B.GS_STAGE_BIN_SORT, -1, 10, 64, 64) == 0


def test_host_argument_checks_need_no_device(lib):
    cam = B.GsCamera()
    cam.width, cam.height, cam.tile = 64, 64, 8  # tile must be 16
    rc = lib.gs_preprocess_fwd(ctypes.byref(cam), 0, *([None] * 11), None, 0, None)
    assert rc == B.GS_ERR_INVALID_ARG
    cam.tile = 16
    rc = lib.gs_render_fwd(ctypes.byref(cam), *([None] * 9), 0, None)
    assert rc == B.GS_ERR_INVALID_ARG
    rc = lib.gs_bin_sort(ctypes.byref(cam), -1, None, None, None, None, 0, None, None, None, None, 0, None)
    assert rc == B.GS_ERR_INVALID_ARG


def test_mask_and_range_buffer_checks_need_no_device(lib):
    """The contribution mask must hold the dispatch-order block plus at least
    one group of bits and be a multiple of 4 words; tile ranges must be
    8-byte aligned.  Both are rejected before anything is enqueued (host
    arrays stand in for device buffers: nothing is dereferenced)."""
    import numpy as np
    cam = B.GsCamera()
    cam.width, cam.height, cam.tile = 64, 48, 16
    T = 4 * 3
    buf = np.zeros(1 << 16, np.uint64)  # 8-byte aligned host storage
    p = lambda off: ctypes.c_void_p(buf.ctypes.data + off)
    need = B.order_words(T) + 4
    assert need == 12 * T + 256 + 4
    for words in (need - 4, need + 2, 0):
        rc = lib.gs_render_fwd(ctypes.byref(cam), p(0), p(0), p(0), p(0), p(0), p(0), p(0), p(0), p(0), words, None)
        assert rc == B.GS_ERR_INVALID_ARG, words
        rc = lib.gs_render_bwd(ctypes.byref(cam), 0, p(0), p(0), p(0), p(0), p(0), p(0), p(0), p(0), words, p(0),
                               None, None, None, None)
        assert rc == B.GS_ERR_INVALID_ARG, words
    assert B.mask_words(100, T) == B.order_words(T) + 4 * 4
    ws_bytes = B.gs_workspace_bytes(B.GS_STAGE_BIN_SORT, 0, 0, cam.width, cam.height)
    ws = np.zeros(ws_bytes + 512, np.uint8)
    ws_p = ctypes.c_void_p((ws.ctypes.data + 255) // 256 * 256)
    rc = lib.gs_bin_sort(ctypes.byref(cam), 0, None, None, None, p(0), 0, None, p(4), None, ws_p, ws_bytes, None)
    assert rc == B.GS_ERR_INVALID_ARG
