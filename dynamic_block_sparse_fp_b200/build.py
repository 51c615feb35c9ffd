"""Compile the CUDA sources into the in-tree shared library ``libfp.so``.

sm_100a only (tcgen05 / TMEM / TMA); the CUDA runtime is linked statically
and only the ``fp_*`` symbols of ``include/fp.h`` are exported.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(HERE, "..", "include", "*.h")) + [os.path.join(CSRC, "exports.map")]
    return all(os.path.getmtime(p) <= t for p in deps)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    """Build libfp.so next to this file; returns its path."""
    if not force and up_to_date():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    # one temporary per process: ranks that find the library stale at the same
    # time each build their own copy, and the atomic rename keeps a whole one
    tmp = f"{LIB}.tmp.{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *(extra or []), "-shared", "-o", tmp, *sources(),
           "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None))
