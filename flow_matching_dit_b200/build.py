"""In-tree build of the CUDA library ``libgdit.so`` for sm_100a.

``python -m flow_matching_dit_b200.build`` (or ``build()``) compiles
``csrc/gdit.cu`` with nvcc into ``flow_matching_dit_b200/libgdit.so``, and
with ``checked=True`` into ``libgdit_checked.so``, the range-checked build
(``-DGDIT_CHECKED=1``: guard bands around device allocations, index checks in
the kernels).  nvcc cross-compiles, so this works on a machine without a GPU.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libgdit.so")
LIB_CHECKED = os.path.join(PKG, "libgdit_checked.so")
SOURCES = sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")) + glob.glob(os.path.join(PKG, "csrc", "*.cuh")))
HEADER = os.path.join(ROOT, "include", "gdit.h")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libgdit.so")


def command(out: str = LIB, checked: bool = False) -> list:
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "-Xcompiler", "-fPIC", "-shared", "-I" + os.path.join(ROOT, "include"),
            "-diag-suppress", "177"] + (["-DGDIT_CHECKED=1"] if checked else []) + \
        ["-o", out, os.path.join(PKG, "csrc", "gdit.cu")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in SOURCES + [HEADER])


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    LIB_OUT = LIB_CHECKED if checked else LIB
    if not force and up_to_date(LIB_OUT):
        return LIB_OUT
    tmp = LIB_OUT + ".tmp"
    cmd = command(tmp, checked)
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    os.replace(tmp, LIB_OUT)
    return LIB_OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, checked="--checked" in sys.argv))
