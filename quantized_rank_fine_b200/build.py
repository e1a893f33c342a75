"""Build libqlora.so in-tree with nvcc for sm_100a.

    python -m quantized_rank_fine_b200.build [--verbose-ptxas]

Each CUDA source is compiled to an object under ``quantized_rank_fine_b200/_build``
and linked, with the CUDA runtime linked statically, into
``quantized_rank_fine_b200/libqlora.so``.  Objects are rebuilt when their source or
any header is newer.  No fast-math: the quantiser and the dequantiser rely on
IEEE binary32 division, products and conversions.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libqlora.so")
SOURCES = ["api.cu", "quantize.cu", "dequant.cu", "skinny.cu", "gemm.cu", "gemv.cu", "xa_small.cu", "noalloc.cu",
           "intq.cu", "selftest.cu"]
HEADERS = ["common.cuh", "kernels.h", "sm100.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--ptxas-options=--warn-on-spills"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newest_dep() -> float:
    paths = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "qlora.h"),
                                                         os.path.abspath(__file__)]
    return max(os.path.getmtime(p) for p in paths if os.path.exists(p))


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    dep = _newest_dep()
    objs = []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(o)
        if not force and os.path.exists(o) and os.path.getmtime(o) >= max(os.path.getmtime(s), dep):
            continue
        cmd = [nvcc(), *ARCH, *FLAGS, "-I", os.path.join(ROOT, "include"), "-c", s, "-o", o]
        if verbose_ptxas:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        tmp = LIB + ".tmp"
        subprocess.run([nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs], check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose_ptxas="--verbose-ptxas" in sys.argv, force="--force" in sys.argv))
