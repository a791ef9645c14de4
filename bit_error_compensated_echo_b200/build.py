"""Build the sm_100a shared library (libecho_b200.so) in-tree with nvcc.

    python -m bit_error_compensated_echo_b200.build

cudart is linked statically, so the library carries its own runtime and
shares the device's primary context with PyTorch.  No fast-math and
-fmad=false: every fp32 operation rounds once, as the definition says.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libecho_b200.so")

COMPILE_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-fmad=false",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
]
LINK_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static"]
BUILD_DIR = os.path.join(PKG, "_build")


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu under csrc/ (one nvcc per translation unit, in
    parallel) and link them into libecho_b200.so (skips if fresh)."""
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    tag = "%d" % os.getpid()
    jobs = []
    for src in sources():
        obj = os.path.join(BUILD_DIR, os.path.basename(src) + "." + tag + ".o")
        cmd = [nvcc(), *COMPILE_FLAGS, "-I" + INCLUDE, "-I" + CSRC, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        jobs.append((obj, subprocess.Popen(cmd)))
    failed = [obj for obj, proc in jobs if proc.wait() != 0]
    objs = [obj for obj, _ in jobs]
    try:
        if failed:
            raise subprocess.CalledProcessError(1, "nvcc -c " + " ".join(failed))
        tmp = LIB + ".tmp" + tag
        cmd = [nvcc(), *LINK_FLAGS, "-o", tmp, *objs]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    finally:
        for obj in objs:
            if os.path.exists(obj):
                os.remove(obj)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
