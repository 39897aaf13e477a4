"""Builds libwoq.so in-tree with nvcc for sm_100a (cross-compiles without a GPU)."""

from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libwoq.so")

CU_SOURCES = ["api.cu", "qgemv.cu", "qgemv_tc.cu", "qgemv_i8tc.cu", "qgemv_chain.cu", "qgemm_tc.cu", "qgemm_noalloc.cu"]
CXX_SOURCES = ["qpack.cpp"]
HEADERS = ["ptx.cuh", "woq_internal.h", "gemv_math.cuh"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-I", INCLUDE, "-I", CSRC, "-Xcompiler", "-fPIC"]


def _stale(out: str, deps: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, force: bool = False) -> str:
    """Compile every source (in parallel) and link libwoq.so; returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    hdr = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "woq.h")]
    jobs, objs = [], []
    for src in CU_SOURCES + CXX_SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src + ".o")
        objs.append(obj)
        if not force and not _stale(obj, [path] + hdr):
            continue
        if src.endswith(".cu"):
            cmd = [NVCC, *ARCH, *COMMON, "-Xptxas", "-v", "-c", path, "-o", obj]
        else:
            cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-I", INCLUDE, "-fno-fast-math", "-c", path, "-o", obj]
        log = open(os.path.join(BUILD, src + ".log"), "w")
        jobs.append((src, subprocess.Popen(cmd, stdout=log, stderr=subprocess.STDOUT), log))
    failed = []
    for src, p, log in jobs:
        rc = p.wait()
        log.close()
        if rc != 0 or verbose:
            with open(log.name) as f:
                sys.stderr.write(f.read())
        if rc != 0:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}; logs in {BUILD}")
    if force or jobs or _stale(LIB, objs):
        cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs, "-lpthread"]
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force="-f" in sys.argv))
