"""Builds ``libfp8w8a8.so`` in-tree with nvcc for sm_100a.

Usage: ``python fp8_w8a8_linear_b200/build.py [--verbose-ptxas]``. nvcc
cross-compiles, so this runs without a GPU. The script is self-contained and
is loaded by file path, never through the package, whose
``__init__`` needs the compiled library to exist already.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp8w8a8.so")
SOURCES = ["fp8w8a8.cu"]
DEPS = ["fp8w8a8.cu", "ptx.cuh", "quant.cuh", "gemm.cuh", "moe.cuh", "act.cuh", "w4a16.cuh"]
HEADER = os.path.join(os.path.dirname(HERE), "include", "fp8w8a8.h")


def nvcc_path() -> str:
    for c in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in DEPS] + [HEADER, __file__]
    return any(os.path.getmtime(p) > t for p in deps)


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [
        nvcc_path(),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
        "-o", LIB + ".tmp",
    ] + [os.path.join(CSRC, s) for s in SOURCES]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libfp8w8a8.so")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose_ptxas="--verbose-ptxas" in sys.argv, force=True))
