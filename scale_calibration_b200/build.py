"""Builds liblh.so (the CUDA library behind include/lh.h) for sm_100a.

    python scale_calibration_b200/build.py [--verbose] [--counters]

The library links the CUDA runtime statically and reaches the driver only
through cudaGetDriverEntryPoint, so it loads (and can be inspected) on a
machine without a GPU driver.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblh.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


# The measurement build: the same sources with the sweep's work counters compiled in
# (see lh_debug_sweep_counts); the bench reads them beside the timed library. Never
# loaded by the package itself.
COUNTERS_LIB = os.path.join(PKG, "liblh_counters.so")


def _stale_lib(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def _build_lib(lib: str, objdir: str, defines: list[str], verbose: bool) -> str:
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *defines, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-cudart", "static", *objs, "-o", tmp])
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale_lib(LIB):
        return LIB
    return _build_lib(LIB, os.path.join(PKG, "_build"), [], verbose)


def build_counters(force: bool = False) -> str:
    if not force and not _stale_lib(COUNTERS_LIB):
        return COUNTERS_LIB
    return _build_lib(COUNTERS_LIB, os.path.join(PKG, "_build_counters"), ["-DLH_SWEEP_COUNTERS=1"], False)


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
    if "--counters" in sys.argv:
        print(build_counters(force=True))
