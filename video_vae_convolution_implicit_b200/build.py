"""Build libconv3d.so (the CUDA library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libconv3d.so")
SOURCES = [os.path.join(CSRC, "conv3d_api.cu"), os.path.join(CSRC, "groupnorm.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("conv3d_kernel.cuh", "wgrad_kernel.cuh", "ptx.cuh")] + [
    os.path.join(ROOT, "include", "conv3d.h")]


def nvcc_command(out: str = LIB, extra=()) -> list[str]:
    return ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
            "-std=c++17", "--shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-I", os.path.join(ROOT, "include"), "-I", CSRC, *extra, "-o", out, *SOURCES]


def build(force: bool = False, verbose: bool = False) -> str:
    stale = not os.path.exists(LIB) or any(os.path.getmtime(d) > os.path.getmtime(LIB) for d in DEPS)
    if force or stale:
        cmd = nvcc_command(extra=("-Xptxas", "-v") if verbose else ())
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
