"""Build the CUDA library ``libdg.so`` in-tree with nvcc for sm_100a.

Run ``python moe_grouped_gemm_09_b200/build.py`` (or call ``build()``; load this
file by path, since importing the package loads the library it builds).  Each
translation unit under ``csrc/`` is compiled on its own (in parallel: the
kernel instantiations of each launch form sit in a unit of their own), then
the objects are linked into one shared library written next to this file so
that it ships with the source tree.  The library links the CUDA runtime
statically and reaches the driver's tensor-map encoder through
``cudaGetDriverEntryPoint``, so loading it needs no GPU.  The ptxas report
(registers, spills, shared memory per kernel) of the last build is kept in
``_build/ptxas.log`` at the repository root.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdg.so")
OBJ_DIR = os.path.join(ROOT, "_build", "obj")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xptxas", "-v"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + [os.path.join(ROOT, "include", "dg.h")])


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _inputs())


def _compile(src: str) -> tuple[str, subprocess.CompletedProcess]:
    obj = os.path.join(OBJ_DIR, os.path.basename(src)[:-3] + ".o")
    r = subprocess.run([NVCC, *COMPILE_FLAGS, "-c", src, "-o", obj], capture_output=True, text=True)
    return obj, r


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    srcs = sources()
    with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        results = list(ex.map(_compile, srcs))
    log = []
    for src, (obj, r) in zip(srcs, results):
        log.append(f"==== {os.path.basename(src)}\n{r.stdout}{r.stderr}")
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"nvcc failed compiling {os.path.basename(src)}")
    with open(os.path.join(ROOT, "_build", "ptxas.log"), "w") as f:
        f.write("\n".join(log))
    objs = [obj for obj, _ in results]
    r = subprocess.run([NVCC, *ARCH, "-shared", *objs, "-o", LIB + ".tmp"],
                       capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed linking libdg.so")
    if verbose:
        sys.stderr.write("\n".join(log))
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
