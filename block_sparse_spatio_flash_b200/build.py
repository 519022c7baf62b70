"""Build libsvgattn.so (sm_100a) in-tree with nvcc.

    python -m block_sparse_spatio_flash_b200.build [--verbose]

Produces block_sparse_spatio_flash_b200/lib/libsvgattn.so and, with build(checked=True), the
checked build lib/libsvgattn_checked.so (-DSVG_CHECKED=1: device-side bounds checks that count
failures instead of trapping; loaded when SVG_CHECKED=1 is set, see svg.py). The libraries link the
CUDA runtime statically and depend on no torch symbol; nvcc cross-compiles them on a machine
without a GPU.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libsvgattn.so")
LIB_CHECKED = os.path.join(LIBDIR, "libsvgattn_checked.so")
SOURCES = ["svg_api.cu", "svg_tilemap.cu", "svg_permute.cu", "svg_attention.cu", "svg_route.cu"]
HEADERS = ["svg_common.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "svg.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    if not force and not _stale(lib):
        return lib
    os.makedirs(LIBDIR, exist_ok=True)
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-I", os.path.join(ROOT, "include"), "-o", lib + ".tmp"]
    if checked:
        cmd += ["-DSVG_CHECKED=1"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv, checked="--checked" in sys.argv))
