"""Build libm3.so (the CUDA kernels + C ABI) in-tree for sm_100a.

    python -m selective_state_space_53_b200.build [--force] [--ptxas-v]

nvcc cross-compiles without a GPU.  Each .cu file is compiled to an object in
parallel (objects under _build/, rebuilt when the file or a header changes), then
the objects are linked into one shared library.  The library links the CUDA
runtime statically, so loading it needs no CUDA toolkit at run time.
"""

from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libm3.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-Xptxas", "-warn-spills",
         "-I", os.path.join(ROOT, "include")]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(ROOT, "include", "m3.h")]


def deps():
    return sources() + headers()


def _obj(src):
    return os.path.join(OBJ, os.path.basename(src)[:-3] + ".o")


def _compile(src, extra, verbose):
    out = _obj(src)
    tmp = out + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", "-o", tmp, src]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    newest_header = max(os.path.getmtime(h) for h in headers())
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(d) <= t for d in deps()):
            return LIB
    os.makedirs(OBJ, exist_ok=True)
    stale = [s for s in sources() if force or extra or not os.path.exists(_obj(s))
             or os.path.getmtime(_obj(s)) < max(os.path.getmtime(s), newest_header)]
    workers = max(1, min(len(stale), os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(workers) as pool:
        for f in [pool.submit(_compile, s, list(extra), verbose) for s in stale]:
            f.result()
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *[_obj(s) for s in sources()]]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
    print(LIB)
