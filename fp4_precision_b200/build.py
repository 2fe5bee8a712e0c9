"""Build the sm_100a CUDA library ``libqfp4.so`` in place (nvcc cross-compiles
without a GPU). Used by ``__graft_entry__.build()`` and by the binding when
the library is missing or older than its sources."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libqfp4.so")
# the same library with every kernel store address checked (QFP4_BOUNDS_CHECK):
# a store outside its buffer is dropped and reported by qfp4_status
LIB_BOUNDS_CHECK = os.path.join(HERE, "libqfp4_bc.so")
SOURCES = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")) + glob.glob(os.path.join(HERE, "csrc", "*.cuh"))
                 + glob.glob(os.path.join(HERE, "csrc", "*.h")) + [os.path.join(ROOT, "include", "qfp4.h")])

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--fmad=false",            # no fused multiply-add: every fp32 step rounds as the method states
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-warn-spills",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in SOURCES)


def build(force: bool = False, verbose: bool = False, bounds_check: bool = False) -> str:
    lib = LIB_BOUNDS_CHECK if bounds_check else LIB
    if not force and not stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), os.path.join(HERE, "csrc", "qfp4_lib.cu"),
           "-o", tmp]
    if bounds_check:
        cmd[1:1] = ["-DQFP4_BOUNDS_CHECK"]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose="-v" in sys.argv, bounds_check="--bounds-check" in sys.argv))
