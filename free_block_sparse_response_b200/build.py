"""Compile the SparsePR CUDA library for sm_100a into this package directory.

``python -m free_block_sparse_response_b200.build`` (or ``build()``) runs one nvcc
invocation over csrc/*.cu and writes ``libsparsepr.so`` next to this file.  A rebuild
is skipped when the library is newer than every source and header.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
REPO_DIR = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_PATH = os.path.join(PKG_DIR, "libsparsepr.so")
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the SparsePR library needs the CUDA toolkit to build")


def _sources():
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = srcs + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(REPO_DIR, "include", "sparsepr.h"), os.path.abspath(__file__)]
    return srcs, deps


def build(force: bool = False, verbose: bool = False) -> str:
    srcs, deps = _sources()
    if not force and os.path.exists(LIB_PATH):
        lib_time = os.path.getmtime(LIB_PATH)
        if all(os.path.getmtime(p) <= lib_time for p in deps):
            return LIB_PATH
    tmp = LIB_PATH + ".tmp"
    cmd = [_nvcc(), "-std=c++17", "-O3", "-lineinfo", *ARCH_FLAGS, "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-shared", "-o", tmp,
           f"-I{os.path.join(REPO_DIR, 'include')}", *srcs]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose:
        print(res.stderr, file=sys.stderr)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
