"""Build the CUDA library (sm_100a) in-tree: _lib/libtriattn.so.

nvcc cross-compiles for sm_100a without a GPU.  The library links the CUDA
runtime statically and resolves the driver (libcuda) at run time, so it also
loads on a machine without a GPU (every call that needs a device then
returns TRI_ATTN_ERR_NO_DEVICE).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_DIR = os.path.join(HERE, "_lib")
LIB = os.path.join(LIB_DIR, "libtriattn.so")
SOURCES = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")) +
                 glob.glob(os.path.join(HERE, "csrc", "*.cuh")) +
                 glob.glob(os.path.join(ROOT, "include", "*.h")))

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in SOURCES)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-I" + os.path.join(ROOT, "include"),
           os.path.join(HERE, "csrc", "tri_attn.cu"), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
