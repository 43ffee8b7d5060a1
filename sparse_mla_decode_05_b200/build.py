"""Builds the sm_100a shared library in-tree.

    python -m sparse_mla_decode_05_b200.build [--verbose]

Produces sparse_mla_decode_05_b200/libsparse_mla.so from csrc/sparse_mla.cu
with nvcc (-gencode arch=compute_100a,code=sm_100a, static CUDA runtime).
No GPU is needed to build.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "sparse_mla.cu")
LIB = os.path.join(PKG, "libsparse_mla.so")
INCLUDE = os.path.join(ROOT, "include")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build_library(verbose: bool = False, extra: list[str] | None = None, out: str = LIB) -> str:
    cmd = [
        nvcc_path(), "-O3", "-std=c++17", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
        "-I", INCLUDE, SRC, "-o", out,
    ]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if extra:
        cmd[1:1] = extra
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    return out


if __name__ == "__main__":
    build_library(verbose="--verbose" in sys.argv)
    print(LIB)
