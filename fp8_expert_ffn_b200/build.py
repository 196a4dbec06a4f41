"""In-tree build of libfp8moe.so (sm_100a) with nvcc, and of its
bounds-checked variant libfp8moe_checked.so (-DMOE_CHECKS: kernels test the
row indices that come from their inputs and flag MOE_STATUS_BOUNDS instead
of accessing out of bounds; the binding loads it when FP8MOE_CHECKED=1).

    python -m fp8_expert_ffn_b200.build [--force] [--verbose-ptxas] [--checked]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp8moe.so")
LIB_CHECKED = os.path.join(HERE, "libfp8moe_checked.so")
BUILD_DIR = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-cudart", "shared",
         "--expt-relaxed-constexpr", "-Werror", "all-warnings", "-Xcompiler", "-fvisibility=hidden"]


PER_FILE = {}


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(os.path.dirname(HERE), "include", "*.h"))


def lib_path(checked: bool = False) -> str:
    return LIB_CHECKED if checked else LIB


def stale(checked: bool = False) -> bool:
    lib = lib_path(checked)
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, verbose_ptxas: bool = False, checked: bool = False) -> str:
    lib = lib_path(checked)
    if not force and not stale(checked):
        return lib
    bdir = BUILD_DIR + ("_checked" if checked else "")
    os.makedirs(bdir, exist_ok=True)
    objs = []
    extra = (["-Xptxas", "-v"] if verbose_ptxas else []) + (["-DMOE_CHECKS"] if checked else [])
    for src in sources():
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *PER_FILE.get(os.path.basename(src), []), *extra, "-c", src, "-o", obj]
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-cudart", "shared", *objs, "-o", tmp])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    path = build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv,
                 checked="--checked" in sys.argv)
    print(path)
