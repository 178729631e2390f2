"""Build the kron_gptq CUDA library (libkrongptq.so) in-tree for sm_100a.

    python -m two_sided_gptq_02_b200.build [--force] [--verbose]
    python -m two_sided_gptq_02_b200.build --define KG_TEST_HANDOFF_FAULT --out <path>.so

Each .cu under csrc/ is compiled separately (so an unchanged file is not rebuilt) and the
objects are linked into a shared library next to this file.  Flags: sm_100a only,
-O3, -lineinfo; no fast-math (rounding decisions must follow IEEE semantics).
A variant (--define NAME, repeatable) is built into the library named by --out, with its objects
in a folder of their own, and leaves the default library alone; the binding loads it when
KRON_GPTQ_LIB names it.
"""
from __future__ import annotations

import argparse
import concurrent.futures
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


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          out: str | None = None) -> str:
    lib = os.path.abspath(out) if out else LIB
    if lib == LIB and any(f.startswith("-D") for f in (extra or [])):
        raise ValueError("a variant build (-D...) needs its own library path (out=...)")
    # objects of a variant live beside its library, so that the default objects are never mixed in
    objdir = BUILD if lib == LIB else os.path.splitext(lib)[0] + "_objs"
    os.makedirs(objdir, exist_ok=True)
    # objects built with other flags are stale (the stamp is written once every object is built)
    stamp, flags = os.path.join(objdir, "flags.txt"), " ".join(CFLAGS + (extra or []))
    if not os.path.exists(stamp):
        force = True
    else:
        with open(stamp) as f:
            force = force or f.read() != flags
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    objs, jobs = [], []
    changed = force or not os.path.exists(lib)
    for src in srcs:
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        newest = max(os.path.getmtime(d) for d in _deps(src))
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < newest:
            cmd = [NVCC, *ARCH, *CFLAGS, *(extra or []), "-I", INCLUDE, "-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), flush=True)
            jobs.append(cmd)
    if jobs:
        # one nvcc per translation unit, in parallel
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as pool:
            for f in [pool.submit(subprocess.check_call, cmd) for cmd in jobs]:
                f.result()
        changed = True
    with open(stamp, "w") as f:
        f.write(flags)
    if changed:
        tmp = lib + f".{os.getpid()}.tmp"
        # cuBLAS (the dense products of the anti-diagonal baseline only) is linked dynamically; a
        # process that imported torch first already holds a libcublas.so.12 and the loader reuses it
        subprocess.check_call([NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-lcublas",
                               "-Xlinker", "-rpath", "-Xlinker", CUDA_LIB])
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--define", action="append", default=[], help="preprocessor macro of a variant build")
    ap.add_argument("--out", default=None, help="library path of a variant build")
    a = ap.parse_args()
    if a.define and not a.out:
        ap.error("a variant (--define) needs its own --out library path")
    print(build(force=a.force, verbose=a.verbose, extra=[f"-D{d}" for d in a.define], out=a.out))
    sys.exit(0)
