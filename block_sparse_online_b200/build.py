"""Build libsolattn.so (sm_100a) in-tree with nvcc.

    python -m block_sparse_online_b200.build [--verbose] [--debug]

The library is written next to this file so that it travels with the source
tree; the Python binding loads it from there.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsolattn.so")
# The same library with the kernels' device-side bounds checks compiled in (-DSOLATTN_DEBUG):
# a failed check records SOLATTN_EBOUNDS in the workspace status word instead of touching
# memory out of range. Same exports; load it explicitly (solattn.load_library(DEBUG_LIB)).
DEBUG_LIB = os.path.join(PKG, "libsolattn_debug.so")
SOURCES = ["solattn_api.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(verbose: bool = False, extra=(), debug: bool = False) -> str:
    out = DEBUG_LIB if debug else LIB
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-I", INCLUDE, "-I", CSRC, "-o", out, *[os.path.join(CSRC, s) for s in SOURCES], *extra]
    if debug:
        cmd.insert(1, "-DSOLATTN_DEBUG")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    return out


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
