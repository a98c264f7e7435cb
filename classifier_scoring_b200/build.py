"""Build librmscore.so (the scorer's C-ABI library) in-tree for sm_100a.

    python -m classifier_scoring_b200.build [-v] [--force] [--checked]

Every .cu/.cpp under csrc/ is compiled by nvcc with
``-gencode arch=compute_100a,code=sm_100a`` and linked against the static CUDA
runtime, so the library loads on a machine without a GPU (entry points that
need a device then return RM_E_DEVICE).  --checked builds
librmscore_checked.so instead: the same sources with -DRM_CHECKED, whose
kernels bounds-check the indices they derive from per-call metadata.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ = os.path.join(ROOT, "_build", "obj")
LIB = os.path.join(PKG, "librmscore.so")
LIB_CHECKED = os.path.join(PKG, "librmscore_checked.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3,-Wall",
         "-I", INCLUDE, "--expt-relaxed-constexpr"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) \
        + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]


def up_to_date(lib_path: str = None) -> bool:
    lib_path = lib_path or LIB
    if not os.path.exists(lib_path):
        return False
    t = os.path.getmtime(lib_path)
    return all(os.path.getmtime(p) <= t for p in _deps())


def _compile(src: str, extra, verbose: bool, obj_dir: str) -> str:
    obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False, extra=(), checked: bool = False) -> str:
    """Build librmscore.so, or with checked=True librmscore_checked.so (the
    same sources with -DRM_CHECKED: bounds-checked kernels)."""
    lib_path = LIB_CHECKED if checked else LIB
    obj_dir = OBJ + "_checked" if checked else OBJ
    flags = list(extra) + (["-DRM_CHECKED"] if checked else [])
    if not force and not extra and up_to_date(lib_path):
        return lib_path
    os.makedirs(obj_dir, exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, flags, verbose, obj_dir), srcs))
    tmp = lib_path + ".tmp"
    cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    v = "-v" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else []
    print(build(force="--force" in sys.argv or bool(extra), verbose=v, extra=extra,
                checked="--checked" in sys.argv))
