"""Build the S2O CUDA library in-tree: score_keys_pooled_b200/libs2o.so.

nvcc cross-compiles for sm_100a (B200) without a GPU present.
Usage: python -m score_keys_pooled_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libs2o.so")
SOURCES = ["s2o_api.cu"]
HEADERS = ["s2o_common.cuh", "pool_score.cuh", "score_i8.cuh", "seg_sort.cuh", "seg_sort2.cuh", "sparse_attn.cuh", "sparse_attn2.cuh", "block_truth.cuh", "qperm.cuh"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(verbose_ptxas: bool = False, out: str = LIB) -> list[str]:
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-o", out]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "s2o.h")]
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or not up_to_date():
        tmp = LIB + ".tmp"
        subprocess.run(command(verbose_ptxas, tmp), check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
