"""Builds the C-ABI shared library ``lib/libsvdq_b200.so`` in-tree for sm_100a.

Usage: ``python w4a4_rank_corrected_smooth_b200/build.py [--force]`` (run by path: importing the
package loads the library this script builds).  nvcc cross-compiles,
so this runs on a machine without a GPU.  Objects go to ``_build/`` next to this file.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIBDIR = os.path.join(HERE, "lib")
LIB = os.path.join(LIBDIR, "libsvdq_b200.so")
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
HEADERS = ["ptx.cuh", "layout.h", "kernels.h", "host_prepare.h"]
SOURCES = ["kernels.cu", "w4a16.cu", "svdq_api.cpp", "host_prepare.cpp"]


def _newer(src_paths, dst):
    if not os.path.exists(dst):
        return True
    t = os.path.getmtime(dst)
    return any(os.path.getmtime(p) > t for p in src_paths)


def _run(cmd):
    print("+", " ".join(cmd), flush=True)
    subprocess.check_call(cmd)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    os.makedirs(LIBDIR, exist_ok=True)
    deps = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "svdq.h"), __file__]
    objs = []
    for src in SOURCES:
        sp = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src + ".o")
        objs.append(obj)
        if not force and not _newer([sp] + deps, obj):
            continue
        if src.endswith(".cu"):
            cmd = [NVCC, *ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-c", sp, "-o", obj]
            if verbose_ptxas:
                cmd.insert(1, "-Xptxas=-v")
        else:
            # Host code: no FMA contraction, IEEE division (the quantizer's decisions depend on it).
            cmd = ["g++", "-O3", "-std=c++17", "-fPIC", "-pthread", "-ffp-contract=off", "-fno-fast-math",
                   "-I", os.path.join(CUDA_HOME, "include"), "-c", sp, "-o", obj]
        _run(cmd)
    if force or _newer(objs, LIB):
        _run([NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", LIB, *objs, "-lpthread"])
    return LIB


def clean():
    shutil.rmtree(BUILD, ignore_errors=True)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="--ptxas-v" in sys.argv)
