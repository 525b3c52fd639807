"""Builds libbgtq.so in-tree with nvcc for sm_100a (B200).

    python -m packed_cache_decode_b200.build_lib [--force]

Objects go to ``_build/`` at the repository root; the shared library lands next to
this file so that the Python binding finds it.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "libbgtq.so")
BUILD = os.path.join(ROOT, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3,-Wall", "-I", os.path.join(ROOT, "include")]
SOURCES = ["host_plan.cpp", "abi.cu", "encode.cu", "decode_mma.cu", "noalloc.cu"]
HEADERS = ["bgtq_internal.h", "kernels.h", "encode_body.cuh", "async_copy.cuh"]


def _newer(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "bgtq.h")]
    objs, jobs = [], []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src + ".o")
        objs.append(obj)
        if force or _newer(obj, [path] + hdrs):
            cmd = [NVCC, *ARCH, *COMMON, "-c", path, "-o", obj]
            if src.endswith(".cpp"):
                cmd = ["g++", "-O3", "-std=c++17", "-fPIC", "-Wall", "-I", os.path.join(ROOT, "include"),
                       "-c", path, "-o", obj]
            if verbose and not src.endswith(".cpp"):
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), flush=True)
            jobs.append((cmd, subprocess.Popen(cmd)))  # the sources compile in parallel
    failed = [cmd for cmd, proc in jobs if proc.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    if force or _newer(OUT, objs):
        cmd = [NVCC, *ARCH, "-shared", "-o", OUT, *objs, "-lcudart_static", "-ldl", "-lrt", "-lpthread"]
        subprocess.run(cmd, check=True)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
