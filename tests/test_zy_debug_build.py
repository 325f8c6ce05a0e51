"""The debug build (libgs_debug.so: the same sources with GS_DEBUG, index
checks before every gather by Gaussian id or list position and before every
write of a list entry), run in a child process on the GPU."""
import json
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.gpu
def test_debug_build_checks_are_clean_on_valid_inputs_and_fire_on_tight_limits():
    from differentiable_gaussian_splatting_preprocess_b200 import build as gsbuild
    gsbuild.build(debug=True)
    env = dict(os.environ, GS_LIBRARY="debug")
    r = subprocess.run([sys.executable, os.path.join(HERE, "_debug_build_child.py")], env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res.pop("library") == "libgs_debug.so"
    from differentiable_gaussian_splatting_preprocess_b200 import binding as B
    for cfg, v in res.items():
        assert v["clean"] == 0 and v["status"] == 0, (cfg, v)   # configs 1-4: no failed check
        assert v["matches_oracle"], (cfg, v)                     # and the same results
        assert v["tight"] == B.GS_ERR_INDEX, (cfg, v)            # limits below the real sizes: reported
        assert v["again"] == 0, (cfg, v)                         # real limits again: clean


def test_release_library_has_no_debug_checks():
    """In the release library the debug entry points report
    GS_ERR_UNIMPLEMENTED (host-only call, no GPU needed)."""
    import ctypes
    from differentiable_gaussian_splatting_preprocess_b200 import binding as B
    L = ctypes.CDLL(os.path.join(os.path.dirname(B.__file__), "libgs.so"))
    f = ctypes.c_int(7)
    assert L.gs_debug_read(ctypes.byref(f), 0) == B.GS_ERR_UNIMPLEMENTED and f.value == 0
    assert L.gs_debug_configure(1, 1) == B.GS_ERR_UNIMPLEMENTED
