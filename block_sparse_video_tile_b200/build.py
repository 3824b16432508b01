"""Build libvsa.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m block_sparse_video_tile_b200.build [--force]

The shared library is written next to this file, so it travels with the
source tree.  No GPU is needed to build (nvcc cross-compiles).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
          "-I", INCLUDE, "-I", CSRC]

TARGETS = {
    "libvsa.so": ["libvsa.cu"],            # the product: C ABI of include/vsa.h
    "libvsa_diag.so": ["vsa_diag.cu"],     # bring-up checks used by the tests only
}


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libvsa")
    return cand


def _sources_mtime() -> float:
    paths = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    paths += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, verbose: bool = False, extra=()) -> list:
    """Compile every target; returns the paths of the built libraries."""
    out = []
    newest = _sources_mtime()
    for lib, srcs in TARGETS.items():
        dst = os.path.join(PKG, lib)
        out.append(dst)
        if not force and os.path.exists(dst) and os.path.getmtime(dst) >= newest:
            continue
        cmd = [_nvcc(), *ARCH, *COMMON, *extra, *[os.path.join(CSRC, s) for s in srcs],
               "-o", dst + ".tmp"]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {lib}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)
        os.replace(dst + ".tmp", dst)
    return out


if __name__ == "__main__":
    force = "--force" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    for p in build(force=force or bool(extra), verbose=True, extra=extra):
        print("built", p)
