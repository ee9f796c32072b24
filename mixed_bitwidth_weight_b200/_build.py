"""Build the qgemm shared library in-tree (nvcc, sm_100a only).

The library is one translation unit (csrc/qgemm.cu) compiled into
``libqgemm.so`` next to this file.  The CUDA runtime is linked statically and
the driver is reached through it at run time, so the library loads on a
machine without a GPU (the exported symbols can be checked there).
"""
from __future__ import annotations

import glob
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libqgemm.so")
STAMP = os.path.join(PKG, "libqgemm.stamp")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(ROOT, "include", "qgemm.h")])


def _digest() -> str:
    """Hash of the sources and the flags, independent of where the tree lives
    (flags are hashed with the tree's root replaced by a placeholder), so the
    same sources give the same digest on every machine."""
    h = hashlib.sha1(" ".join(f.replace(ROOT, "<root>") for f in FLAGS).encode())
    for f in _sources():
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile csrc/qgemm.cu into libqgemm.so unless it is up to date."""
    d = _digest()
    if not force and os.path.exists(LIB) and os.path.exists(STAMP):
        with open(STAMP) as f:
            if f.read().strip() == d:
                return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *extra, "-o", tmp, os.path.join(CSRC, "qgemm.cu")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(d)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
