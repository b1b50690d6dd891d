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


# Test build: the same sources with the cooperative fill's grid-barrier wait cut to zero,
# so that an ordinary partition call makes that bounded wait run out (its error path
# records SPARSEPR_ERR_TIMEOUT and returns; no GPU fault, nothing left in flight).
WAITTEST_LIB_PATH = os.path.join(PKG_DIR, "libsparsepr_waittest.so")
VARIANTS = {None: (LIB_PATH, []), "waittest": (WAITTEST_LIB_PATH, ["-DSPR_GRID_WAIT_LIMIT_NS=0ull"])}


def build(force: bool = False, verbose: bool = False, variant=None) -> str:
    lib_path, defines = VARIANTS[variant]
    srcs, deps = _sources()
    if not force and os.path.exists(lib_path):
        lib_time = os.path.getmtime(lib_path)
        if all(os.path.getmtime(p) <= lib_time for p in deps):
            return lib_path
    tmp = lib_path + ".tmp"
    cmd = [_nvcc(), "-std=c++17", "-O3", "-lineinfo", *ARCH_FLAGS, "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-shared", "-o", tmp, *defines,
           f"-I{os.path.join(REPO_DIR, 'include')}", *srcs]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose:
        print(res.stderr, file=sys.stderr)
    os.replace(tmp, lib_path)
    return lib_path


def build_all(force: bool = False) -> None:
    """The library and its wait-limit test build."""
    for variant in VARIANTS:
        build(force=force, variant=variant)


if __name__ == "__main__":
    if "--all" in sys.argv:
        build_all(force="--force" in sys.argv)
    else:
        print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
