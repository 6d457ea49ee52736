"""Build libhadq.so in-tree with nvcc for sm_100a (B200).

Run as ``python -m hadamard_rotation_outlier_b200.build``; ``--verbose`` adds
``-Xptxas -v`` (registers, spills and shared memory per kernel).  The library
is rebuilt when any source under ``csrc/`` or ``include/`` is newer than it.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libhadq.so")
SOURCES = [os.path.join(PKG, "csrc", "hadq_api.cu")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _deps():
    return (glob.glob(os.path.join(PKG, "csrc", "*")) +
            glob.glob(os.path.join(ROOT, "include", "*.h")))


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libhadq.so")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if it is missing or stale; return its path."""
    if not force and not needs_build():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc_path(), "-shared", "-Xcompiler", "-fPIC", "-O3", "-lineinfo", "-std=c++17",
           *ARCH, "-o", tmp, *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stderr[-8000:]}")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
