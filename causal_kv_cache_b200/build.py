"""Build libca2.so in-tree with nvcc for sm_100a (B200), and its bounds-checked debug build
libca2_debug.so (the same sources with -DCA2_DEBUG; select it with CA2_LIBRARY).

    python -m causal_kv_cache_b200.build [--verbose-ptxas] [--release-only]

The library is a plain shared object with an extern "C" surface (include/ca2.h); the
Python binding loads it with ctypes.  The CUDA runtime is linked statically, so the
library loads on a machine without a GPU (only calls that touch the device fail there).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libca2.so")
LIB_DEBUG = os.path.join(PKG, "libca2_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17", "-rdc=true",
    "-Xcompiler", "-fPIC,-O2", "-shared",
    "-Xcudafe", "--diag_suppress=177",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(out: str) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        [os.path.join(ROOT, "include", "ca2.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, out: str = LIB, debug: bool = False) -> str:
    if not force and not _stale(out):
        return out
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include")]
    if debug:
        cmd += ["-DCA2_DEBUG"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    tmp = out + ".tmp%d" % os.getpid()
    cmd += [*sources(), "-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build_debug(force: bool = False) -> str:
    return build(force=force, out=LIB_DEBUG, debug=True)


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
    if "--release-only" not in sys.argv:
        build_debug(force=True)
        print(LIB_DEBUG)
