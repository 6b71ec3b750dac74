"""Build the HISA CUDA library in-tree: hierarchical_top_indexer_b200/libhisa_b200.so.

nvcc for sm_100a only; cudart is linked statically and the driver API is
reached through cudaGetDriverEntryPoint, so the library needs nothing but the
NVIDIA driver at run time.

    python hierarchical_top_indexer_b200/build.py [--verbose-ptxas] [--if-stale]

(run as a script: importing the package itself needs the built library)
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libhisa_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(ROOT, "include", "*.h")))


def stale(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(f) > t for f in sources() + headers())


def build(out: str = LIB, verbose_ptxas: bool = False, extra=(), jobs: int = 8) -> str:
    """Compile every .cu to an object (in parallel), then link the shared library."""
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    common = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
              "-I", os.path.join(ROOT, "include"), *extra]
    if verbose_ptxas:
        common += ["-Xptxas", "-v"]
    procs, objs = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        objs.append(obj)
        procs.append(subprocess.Popen(common + ["-c", src, "-o", obj]))
        while len([p for p in procs if p.poll() is None]) >= jobs:
            procs[0].wait()
    rc = [p.wait() for p in procs]
    if any(rc):
        raise RuntimeError("nvcc failed")
    subprocess.run([NVCC, *ARCH, "-shared", "-o", out, *objs], check=True)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--if-stale", action="store_true")
    a = ap.parse_args(argv)
    if a.if_stale and not stale():
        print(LIB, "(up to date)")
        return 0
    print(build(verbose_ptxas=a.verbose_ptxas))
    return 0


if __name__ == "__main__":
    sys.exit(main())
