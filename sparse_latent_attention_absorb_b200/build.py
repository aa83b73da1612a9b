"""Builds the sm_100a shared library ``libmla_sparse_decode.so`` in-tree.

    python -m sparse_latent_attention_absorb_b200.build

nvcc cross-compiles for sm_100a without a GPU.  The library links the CUDA
runtime statically, so it only needs the NVIDIA driver at run time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libmla_sparse_decode.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
SOURCES = [os.path.join(CSRC, "mla_sparse_decode.cu"), os.path.join(CSRC, "selftest.cu")]
DEPENDS = SOURCES + [os.path.join(CSRC, f) for f in ("kernels.cuh", "ptx.cuh", "projection.cuh", "projection_plan.h", "index_check.cuh", "dequant.cuh")] + [
    os.path.join(INCLUDE, "mla_sparse_decode.h")]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str, verbose_ptxas: bool = False) -> list[str]:
    cmd = [nvcc(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-o", out, *SOURCES]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def is_stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(p) > t for p in DEPENDS)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or is_stale():
        tmp = LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.run(command(tmp, verbose_ptxas), check=True)
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
    print(LIB_PATH)
