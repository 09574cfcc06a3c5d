"""Builds libug.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: ``python -m block_sparse_local_raster_b200.build [--force] [--verbose] [--debug]``.
Objects go to ``_build/`` next to this file, the library to ``libug.so`` next
to this file.  Rebuilds only what is older than its sources or headers.

``--debug`` builds ``libug_debug.so`` (objects in ``_build_debug/``) with
``-DUG_DEBUG=1``: the same kernels with a range check before every global
access whose index they compute (see csrc/ug_debug.h).  The GPU tests run the
small geometries through it.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libug.so")
BUILD_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libug_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "--expt-relaxed-constexpr",
          # Host code: no fast-math; keep libm cos/sin calls separate.
          "-Xcompiler", "-fPIC,-fno-builtin-sin,-fno-builtin-cos,-fno-fast-math",
          "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _newer(src_paths, target) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in src_paths)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    bdir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD, LIB)
    flags = CFLAGS + (["-DUG_DEBUG=1"] if debug else [])
    os.makedirs(bdir, exist_ok=True)
    headers = (glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
               + glob.glob(os.path.join(INCLUDE, "*.h")))
    objs = []
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _newer([src] + headers, obj):
            cmd = [nvcc()] + ARCH + flags + (["-Xptxas", "-v"] if verbose else []) + \
                ["-c", src, "-o", obj]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if verbose or r.returncode:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode:
                raise RuntimeError(f"nvcc failed on {os.path.basename(src)}")
    if force or _newer(objs, lib):
        cmd = [nvcc()] + ARCH + ["-shared", "-o", lib + ".tmp"] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("link failed")
        os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--debug", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, debug=a.debug))
