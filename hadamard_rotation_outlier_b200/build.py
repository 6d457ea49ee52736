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
SOURCES = sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))
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


def _compile(src: str, obj: str, verbose: bool):
    cmd = [nvcc_path(), "-c", "-Xcompiler", "-fPIC", "-O3", "-lineinfo", "-std=c++17", *ARCH,
           "-o", obj, src]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return subprocess.run(cmd, capture_output=True, text=True)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if it is missing or stale; return its path.

    Each kernel family is its own translation unit; they compile in parallel
    and link into one shared library.
    """
    if not force and not needs_build():
        return LIB
    from concurrent.futures import ThreadPoolExecutor

    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = [os.path.join(objdir, os.path.basename(src)[:-3] + ".o") for src in SOURCES]
    with ThreadPoolExecutor(len(SOURCES)) as ex:
        results = list(ex.map(lambda so: _compile(so[0], so[1], verbose), zip(SOURCES, objs)))
    for src, res in zip(SOURCES, results):
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)} ({res.returncode}):\n"
                               f"{res.stderr[-8000:]}")
        if verbose:
            sys.stderr.write(res.stderr)
    tmp = LIB + ".tmp"
    res = subprocess.run([nvcc_path(), "-shared", *ARCH, "-o", tmp, *objs], capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc link failed ({res.returncode}):\n{res.stderr[-8000:]}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
