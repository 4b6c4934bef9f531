"""Build libulysses_a2a.so in-tree with nvcc for sm_100a.

Usage: ``python sequence_all_re_b200/build.py [--force] [--ptxas-info]``.
The library is linked against the static CUDA runtime and reaches the driver
API through ``cudaGetDriverEntryPointByVersion``, so it loads (and exports its
symbols) on a machine without a GPU driver; only its compute calls need one.
"""

from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libulysses_a2a.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def stale(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, ptxas_info: bool = False, out: str = LIB) -> str:
    if not force and not stale(out):
        return out
    cmd = [nvcc(), *ARCH, "-lineinfo", "-O3", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC,-O2,-Wall", "-I", INCLUDE, "-I", CSRC,
           "-o", out, *sorted(glob.glob(os.path.join(CSRC, "*.cu")))]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force or a.ptxas_info, ptxas_info=a.ptxas_info))
