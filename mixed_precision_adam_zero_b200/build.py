"""Build libzero_adam.so in-tree with nvcc for sm_100a (B200)."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SOURCES = [os.path.join(PKG, "csrc", "zero_adam_api.cu"), os.path.join(PKG, "csrc", "zero_adam_host.cpp"),
           os.path.join(PKG, "csrc", "zero_adam_ckpt.cpp")]
DEPS = SOURCES + [os.path.join(PKG, "csrc", "zero_adam_kernels.cuh"), os.path.join(PKG, "csrc", "zero_adam_bulk.cuh"),
                  os.path.join(PKG, "csrc", "zero_adam_internal.h"), os.path.join(ROOT, "include", "zero_adam.h")]
OUT = os.path.join(PKG, "libzero_adam.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library unless it is newer than every source; return its path."""
    if not force and os.path.exists(OUT):
        built = os.path.getmtime(OUT)
        if all(os.path.getmtime(d) <= built for d in DEPS):
            return OUT
    tmp = OUT + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-o", tmp, *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
