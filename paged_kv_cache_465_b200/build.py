"""Builds libpagedattn.so in-tree with nvcc for sm_100a (no JIT cache, no torch extension).

    python paged_kv_cache_465_b200/build.py [-v]

The CUDA sources are compiled as one translation unit (pagedattn.cu includes the kernel
headers), the host allocator separately; the CUDA runtime is linked statically so the
library has no dependency on the process's libcudart.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libpagedattn.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = _sources() + [os.path.join(INCLUDE, "pagedattn.h"), __file__]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, extra=None) -> str:
    if not force and not _stale():
        return LIB
    nvcc = _nvcc()
    os.makedirs(BUILD, exist_ok=True)
    common = ["-O3", "-std=c++17", "-I", INCLUDE, "-I", CSRC, "-Xcompiler", "-fPIC"]
    cu_obj = os.path.join(BUILD, "pagedattn.o")
    cpp_obj = os.path.join(BUILD, "allocator.o")
    cmds = [
        [nvcc, *ARCH, "-lineinfo", *common, "-Xptxas", "-v" if verbose else "-O3",
         "-c", os.path.join(CSRC, "pagedattn.cu"), "-o", cu_obj] + list(extra or []),
        [nvcc, *common, "-Wno-deprecated-gpu-targets", "-x", "c++", "-c", os.path.join(CSRC, "allocator.cpp"), "-o", cpp_obj],
        [nvcc, *ARCH, "-shared", "-cudart", "static", cu_obj, cpp_obj, "-o", LIB + ".tmp"],
    ]
    for c in cmds:
        r = subprocess.run(c, capture_output=True, text=True)
        if verbose or r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError("build failed: " + " ".join(c))
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
