"""Builds libmuon.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m newton_schulz_norm_b200.build [--force] [--verbose]

The library is plain C++/CUDA with an extern "C" interface (include/muon.h);
it links the CUDA runtime statically and reaches the driver's tensor-map
encoder through cudaGetDriverEntryPoint, so it needs no libcuda at link time.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG_DIR, "libmuon.so")
# The same sources with -DMUON_BOUNDS_CHECK: every kernel validates its table
# entries and reports MUON_ERR_INVALID_ARG instead of reading out of bounds
# (include/muon_debug.h).  For tests; the product path loads LIB_PATH.
CHECKED_LIB_PATH = os.path.join(PKG_DIR, "libmuon_checked.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmuon.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=None, checked: bool = False) -> str:
    """Build libmuon.so (or, with ``checked``, libmuon_checked.so) unless it
    is newer than every source; returns its path."""
    target = CHECKED_LIB_PATH if checked else LIB_PATH
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]
    if not force and not _stale(target, deps):
        return target
    tmp = target + ".tmp"
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-std=c++17", "-lineinfo", "--shared",
           "-Xcompiler", "-fPIC,-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC,
           "-cudart", "static", "-o", tmp, *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if checked:
        cmd[1:1] = ["-DMUON_BOUNDS_CHECK"]
    if extra_flags:
        cmd[1:1] = list(extra_flags)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed building {os.path.basename(target)}:\n" + " ".join(cmd))
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checked", action="store_true", help="the bounds-checked variant")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, checked=a.checked))
