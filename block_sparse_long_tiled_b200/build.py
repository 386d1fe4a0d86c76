"""Build libsskip_attn.so (release) and libsskip_attn_debug.so (device-side
index checks, SSKIP_DEBUG_CHECKS=1) in-tree with nvcc for sm_100a.

    python -m block_sparse_long_tiled_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libsskip_attn.so")
LIB_DEBUG = os.path.join(PKG, "libsskip_attn_debug.so")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared"]


def _sources():
    return (glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
            [os.path.join(ROOT, "include", "sskip_attn.h")])


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale(lib: str) -> bool:
    return not os.path.exists(lib) or any(os.path.getmtime(s) > os.path.getmtime(lib)
                                          for s in _sources())


def build(force: bool = False, verbose: bool = False) -> str:
    """Build both libraries if a source is newer (in parallel); returns the
    release library's path."""
    jobs = []
    for lib, extra in ((LIB, []), (LIB_DEBUG, ["-DSSKIP_DEBUG_CHECKS=1"])):
        if not (force or _stale(lib)):
            continue
        tmp = f"{lib}.tmp{os.getpid()}"
        cmd = [nvcc(), *NVCC_FLAGS, *extra, "-o", tmp, os.path.join(CSRC, "sskip_attn.cu")]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        jobs.append((subprocess.Popen(cmd), tmp, lib, cmd))
    for proc, tmp, lib, cmd in jobs:
        if proc.wait() != 0:
            raise subprocess.CalledProcessError(proc.returncode, cmd)
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
