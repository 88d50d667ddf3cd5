"""Builds libsparsed.so in-tree with nvcc for sm_100a (no GPU needed)."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsparsed.so")
SOURCES = ["sparsed_api.cu"]
DEPS = ["sparsed_api.cu", "attn_kernel.cuh", "attn_list_kernel.cuh", "select_kernels.cuh", "column_kernels.cuh", "losa_kernels.cuh",
        "ptx_sm100.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def nvcc_cmd(out: str = LIB, extra: list[str] | None = None) -> list[str]:
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
            "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I", CSRC,
            *(extra or []), "-o", out, *[os.path.join(CSRC, s) for s in SOURCES]]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    srcs = [os.path.join(CSRC, s) for s in DEPS] + [os.path.join(INCLUDE, "sparsed.h"), __file__]
    return any(os.path.getmtime(s) > t for s in srcs)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or _stale():
        cmd = nvcc_cmd()
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
