"""Builds libnaju.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m discrete_selective_ssm_b200.build [--force]

nvcc compiles every ``csrc/*.cu`` to an object file (in parallel, under
``_build/`` at the repository root) and links them into one shared library
next to this file; the build is skipped when the library is newer than all
sources and headers, and an object is recompiled only when it is older than
its source or any header.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libnaju.so")
OBJDIR = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the Naju CUDA library cannot be built")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h*")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in sources() + _headers())


def _obj(src: str) -> str:
    return os.path.join(OBJDIR, os.path.basename(src)[:-3] + ".o")


def _compile(src: str, force: bool, verbose: bool) -> str:
    obj = _obj(src)
    if not force and os.path.exists(obj):
        t = os.path.getmtime(obj)
        if all(os.path.getmtime(f) <= t for f in [src] + _headers()):
            return obj
    tmp = obj + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-c",
           "-I", INCLUDE, "-I", CSRC, "-o", tmp, src]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, obj)
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    srcs = sources()
    # the largest translation units first, so they do not finish last
    srcs.sort(key=os.path.getsize, reverse=True)
    workers = max(1, min(len(srcs), os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        objs = list(ex.map(lambda f: _compile(f, force, verbose), srcs))
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([_nvcc(), *ARCH, "-shared", "-o", tmp, *sorted(objs)])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
