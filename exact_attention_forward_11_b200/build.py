"""Builds the C-ABI shared library (libattn_b200.so) in-tree with nvcc for sm_100a,
and its debug build (libattn_b200_debug.so: the same sources with -DATTN_DEBUG,
device-side index checks that record ATTN_ERR_BOUNDS and skip the access).

    python -m exact_attention_forward_11_b200.build [--force] [--debug]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libattn_b200.so")
LIB_DEBUG = os.path.join(HERE, "libattn_b200_debug.so")

SOURCES = ["attn_api.cu"]
HEADERS = ["sm100.cuh", "status.cuh", "attn_fwd_kernel.cuh", "attn_fwd1_kernel.cuh", "mxfp8_quant_kernel.cuh", "attn_bwd_kernel.cuh", "fp8_prep_kernel.cuh", "w4a16_kernel.cuh"]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, h) for h in os.listdir(INCLUDE)] + [__file__]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, *(["-DATTN_DEBUG"] if debug else []), "-I" + INCLUDE, "-I" + CSRC, "-o", tmp,
           *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
