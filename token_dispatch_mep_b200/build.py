"""Builds ``libmep.so`` (the CUDA kernels and the C ABI) in-tree with nvcc for
sm_100a.  ``python -m token_dispatch_mep_b200.build`` or ``build()``."""
from __future__ import annotations

import concurrent.futures
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmep.so")
OBJDIR = os.path.join(ROOT, "_build")
SOURCES = ["abi.cu", "plan.cu", "dispatch.cu", "combine.cu", "reduce.cu", "backward.cu", "prefetch.cu",
           "noalloc.cu", "ipc.cu", "barrier.cu", "dispatch_bulk.cu"]
HEADERS = ["mep_device.cuh", "mep_internal.h"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def _stale(out: str, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, extra, objdir: str = OBJDIR) -> str:
    obj = os.path.join(objdir, os.path.splitext(src)[0] + ".o")
    deps = [os.path.join(CSRC, src), os.path.join(INCLUDE, "mep.h")] + \
        [os.path.join(CSRC, h) for h in HEADERS]
    if _stale(obj, deps):
        subprocess.run([NVCC, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj], check=True)
    return obj


def build(verbose_ptxas: bool = False, force: bool = False, defines=(), lib: str = LIB,
          objdir: str = OBJDIR) -> str:
    """Compile every kernel source for sm_100a and link ``libmep.so`` (next to
    this file unless `lib` says otherwise).  `defines` are extra -D tunables
    (launch shapes); the default build uses none.  Returns the library path."""
    os.makedirs(objdir, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    extra += [f"-D{d}" for d in defines]
    if force:
        for f in os.listdir(objdir):
            if f.endswith(".o"):
                os.remove(os.path.join(objdir, f))
    with concurrent.futures.ThreadPoolExecutor(len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, objdir), SOURCES))
    if force or _stale(lib, objs):
        subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-o", lib, *objs], check=True)
    return lib


if __name__ == "__main__":
    print(build(verbose_ptxas="-v" in sys.argv, force="-f" in sys.argv))
