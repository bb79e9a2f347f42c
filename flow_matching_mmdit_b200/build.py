"""Build liblens_dit.so in-tree with nvcc for sm_100a.

    python -m flow_matching_mmdit_b200.build [--force] [--verbose]

LENS_NVCC_EXTRA (environment) adds nvcc flags to every compile, e.g.
LENS_NVCC_EXTRA="-DLENS_ATTN_EMU_MASK=0x5555u" for a measurement build (use --force).

Objects go to flow_matching_mmdit_b200/_build/; the shared library is written next
to this file so it travels with the source tree.  The CUDA runtime is linked
statically and the driver API is reached through cudaGetDriverEntryPoint, so the
library loads on a machine without a GPU (symbols can be inspected there).
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "liblens_dit.so")
INCLUDE = os.path.join(ROOT, "include")

SOURCES = ["lens_dit.cu", "gemm.cu", "attention.cu", "elementwise.cu", "noalloc.cu", "w4.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def _deps() -> list:
    return [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "lens_dit.h")]


def _stale(target: str, deps: list) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    deps = _deps()
    objs = []
    for src in SOURCES:
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, deps):
            extra = os.environ.get("LENS_NVCC_EXTRA", "").split()
            cmd = [nvcc()] + ARCH + FLAGS + extra + (["-Xptxas", "-v"] if ptxas_verbose else []) + [
                "-c", os.path.join(CSRC, src), "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
    if force or _stale(LIB, objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", LIB] + objs + ["-ldl", "-lpthread", "-lrt"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.ptxas_verbose))
    sys.exit(0)
