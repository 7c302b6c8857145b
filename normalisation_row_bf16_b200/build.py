"""Builds libmxnorm_b200.so in-tree with nvcc for sm_100a (no JIT cache).

    python -m normalisation_row_bf16_b200.build
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmxnorm_b200.so")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xptxas", "-warn-spills"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every translation unit in csrc/ (in parallel) and link the library."""
    if not force and not is_stale():
        return LIB
    tus = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    procs = []
    for tu in tus:
        obj = os.path.join(objdir, os.path.basename(tu) + f".{os.getpid()}.o")
        cmd = [nvcc(), *NVCC_FLAGS, "-c", "-I" + INCLUDE, "-o", obj, tu]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((obj, subprocess.Popen(cmd)))
    objs = []
    failed = False
    for obj, p in procs:
        failed |= p.wait() != 0
        objs.append(obj)
    if failed:
        raise RuntimeError("nvcc failed")
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs], check=True)
    os.replace(tmp, LIB)
    for o in objs:
        os.remove(o)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
