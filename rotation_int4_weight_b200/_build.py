"""Builds libparo.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: python rotation_int4_weight_b200/_build.py [--force] [-v] [--timeline]
(run it as a file: importing the package would first load the library it builds)

--timeline builds libparo_timeline.so instead: the same sources compiled with
PARO_TIMELINE, whose fused one-token decode kernel records global-timer stamps
of its phases per CTA (read back by paro_timeline_read; `bench.py --timeline`
loads it and prints the table).  The package loads it in place of libparo.so
when the environment sets PARO_TIMELINE=1.
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
LIB = os.path.join(PKG, "libparo.so")
BUILD_TIMELINE = os.path.join(PKG, "_build_timeline")
LIB_TIMELINE = os.path.join(PKG, "libparo_timeline.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
          "-I", os.path.join(ROOT, "include"), "--expt-relaxed-constexpr"]
# Files whose results must be bit-exact with an IEEE reference compile without FMA contraction.
PER_FILE = {"pack.cu": ["-fmad=false"]}
SOURCES = ["api.cu", "rotate.cu", "rotate_decode.cu", "rotate_backward.cu", "pack.cu", "w4_gemv.cu", "w4_tc.cu", "w4_stream.cu", "plan.cu", "noalloc.cu", "w4a4.cu"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newer(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose: bool = False, timeline: bool = False) -> str:
    build_dir, lib = (BUILD_TIMELINE, LIB_TIMELINE) if timeline else (BUILD, LIB)
    defines = ["-DPARO_TIMELINE=1"] if timeline else []
    os.makedirs(build_dir, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    headers.append(os.path.join(ROOT, "include", "paro.h"))
    objs = []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(obj)
        if not force and _newer(obj, [path] + headers):
            continue
        cmd = [nvcc(), *ARCH, *COMMON, *defines, *PER_FILE.get(src, []), "-c", path, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    if force or not _newer(lib, objs):
        cmd = [nvcc(), *ARCH, "-shared", "-o", lib, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, timeline="--timeline" in sys.argv))
