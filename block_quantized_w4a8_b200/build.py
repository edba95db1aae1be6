"""Builds libw4a8.so in-tree with nvcc for sm_100a (no JIT, no torch extension)."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC_DIR = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libw4a8.so")
CHECKED_LIB = os.path.join(PKG, "libw4a8_checked.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources() -> list[str]:
    out = [os.path.join(ROOT, "include", "w4a8.h")]
    for f in sorted(os.listdir(SRC_DIR)):
        if f.endswith((".cu", ".cuh")):
            out.append(os.path.join(SRC_DIR, f))
    return out


def lib_path(checked: bool = False) -> str:
    return CHECKED_LIB if checked else LIB


def up_to_date(checked: bool = False) -> bool:
    lib = lib_path(checked)
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Compile the library for sm_100a. checked=True builds libw4a8_checked.so with
    -DW4A8_CHECKED: the same kernels with device-side checks of each copy's alignment that
    report W4A8_ERR_CHECK instead of faulting (a stand-in for a memory checker)."""
    lib = lib_path(checked)
    if not force and up_to_date(checked):
        return lib
    cmd = [
        NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
        "-shared", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"),
        os.path.join(SRC_DIR, "w4a8.cu"), "-o", lib + ".tmp", "-lcudart",
    ]
    if checked:
        cmd.insert(1, "-DW4A8_CHECKED")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd, timeout=900)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv, checked="--checked" in sys.argv))
