"""Build ``libgs.so`` (the rasterizer's C-ABI library) in-tree for sm_100a.

Every translation unit under ``csrc/`` is compiled by nvcc for
``arch=compute_100a,code=sm_100a`` with line info, no fast-math, and the CUDA
runtime linked statically, then linked into one shared object beside this
file.  Objects go to ``_build/`` (git-ignored).

``build(debug=True)`` builds ``libgs_debug.so`` from the same sources with
GS_DEBUG defined (index checks before every gather by Gaussian id or list
position; see gs_debug_configure in include/gs.h), as relocatable device code
so that all translation units share one device-side debug word.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT_DIR = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libgs.so")
DEBUG_LIB = os.path.join(HERE, "libgs_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
          "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date(debug: bool = False) -> bool:
    lib = DEBUG_LIB if debug else LIB
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and up_to_date(debug):
        return lib
    out_dir = os.path.join(OUT_DIR, "debug") if debug else OUT_DIR
    extra = ["-DGS_DEBUG", "-rdc=true"] if debug else []
    os.makedirs(out_dir, exist_ok=True)
    objs = []
    for src in sources():
        obj = os.path.join(out_dir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *CFLAGS, *extra, "-c", src, "-o", obj]
        if ptxas_info:
            cmd.insert(1, "-Xptxas=-v")
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, *extra, "-shared", "-cudart", "static", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    dbg = "--debug" in sys.argv
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, ptxas_info="--ptxas" in sys.argv, debug=dbg))
