"""Build the kron_gptq CUDA library (libkrongptq.so) in-tree for sm_100a.

    python -m two_sided_gptq_02_b200.build [--force] [--verbose]

Each .cu under csrc/ is compiled separately (so an unchanged file is not rebuilt) and the
objects are linked into a shared library next to this file.  Flags: sm_100a only,
-O3, -lineinfo; no fast-math (rounding decisions must follow IEEE semantics).
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libkrongptq.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
CUDA_LIB = os.path.join(os.path.dirname(os.path.dirname(NVCC)), "lib64")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
          "-Xcompiler", "-fvisibility=hidden"]


def _deps(src: str) -> list[str]:
    return [src] + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(INCLUDE, "kron_gptq.h")]


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    objs = []
    changed = force or not os.path.exists(LIB)
    for src in srcs:
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        newest = max(os.path.getmtime(d) for d in _deps(src))
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < newest:
            cmd = [NVCC, *ARCH, *CFLAGS, *(extra or []), "-I", INCLUDE, "-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), flush=True)
            subprocess.check_call(cmd)
            changed = True
    if changed:
        tmp = LIB + f".{os.getpid()}.tmp"
        # cuBLAS (the one-sided path's plain GEMM) is linked dynamically; a process that imported
        # torch first already holds a libcublas.so.12 and the loader reuses it
        subprocess.check_call([NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-lcublas",
                               "-Xlinker", "-rpath", "-Xlinker", CUDA_LIB])
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
    sys.exit(0)
