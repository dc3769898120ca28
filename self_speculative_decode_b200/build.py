"""Build libripe.so in-tree with nvcc for sm_100a.

``python -m self_speculative_decode_b200.build`` (or ``build()``) compiles the
CUDA sources under ``csrc/`` into ``self_speculative_decode_b200/lib/libripe.so``;
``build(debug=True)`` compiles the same sources with ``-DRIPE_DEBUG`` into
``lib/libripe_debug.so`` (device-side index checks, dead rows poisoned after every
commit; select it with the environment variable ``RIPE_LIBRARY``).
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
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libripe.so")
LIB_DEBUG = os.path.join(LIBDIR, "libripe_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-use_fast_math", "-Xcompiler", "-fPIC,-O3",
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    os.makedirs(LIBDIR, exist_ok=True)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, *FLAGS, f"-I{INCLUDE}", "-shared", "-o", tmp, *sources()]
    if debug:
        cmd.insert(1, "-DRIPE_DEBUG")
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="-v" in sys.argv, debug="--debug" in sys.argv))
