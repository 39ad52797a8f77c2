"""Builds libcswattn.so in-tree with nvcc for sm_100a.

    python -m causal_sliding_window_rope_b200.build

The CUDA runtime is linked statically and the driver is reached through the
runtime's entry-point query, so the library also loads (without computing) on
a machine that has no GPU driver.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libcswattn.so")
LIB_CHECK = os.path.join(PKG, "libcswattn_check.so")  # CSWATTN_CHECK=1: device-side bounds checks
SOURCES = ["cswattn.cu"]
HEADER = os.path.join(ROOT, "include", "cswattn.h")


def deps() -> list[str]:
    """Every file the library is compiled from: the translation unit, every
    kernel header next to it and the public header."""
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [HEADER, os.path.abspath(__file__)])


NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def stale(lib: str | None = None) -> bool:
    lib = lib or LIB
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in deps())


def build(force: bool = False, verbose: bool = False, check: bool = False) -> str:
    """Compile libcswattn.so (or, with check, libcswattn_check.so: the same
    library with CSWATTN_CHECK=1 device-side bounds checks)."""
    lib = LIB_CHECK if check else LIB
    if not force and not stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"),
           *(["-DCSWATTN_CHECK=1"] if check else []),
           *(os.path.join(CSRC, s) for s in SOURCES), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv, check="--check" in sys.argv))
