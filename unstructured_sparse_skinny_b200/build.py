"""Builds libflashspmm.so in-tree with nvcc for sm_100a.

Usage: ``python -m unstructured_sparse_skinny_b200.build [--force]``.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
SOURCES = [PKG / "csrc" / f for f in ("flashspmm_api.cu", "tcsl_encode.cu", "spmm_lscd.cu", "spmm_noalloc.cu", "partition.cu", "round_f16.cu", "selftest.cu")]
DEPS = SOURCES + [PKG / "csrc" / f for f in ("common.cuh", "sm100_primitives.cuh")] + [ROOT / "include" / "flashspmm.h"]
LIB = PKG / "libflashspmm.so"
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


def nvcc_path() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not Path(p).exists():
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libflashspmm")
    return p


def up_to_date() -> bool:
    if not LIB.exists():
        return False
    t = LIB.stat().st_mtime
    return all(d.stat().st_mtime <= t for d in DEPS)


def build_library(force: bool = False, verbose: bool = False) -> Path:
    if not force and up_to_date():
        return LIB
    tmp = LIB.with_name(f"libflashspmm.so.tmp{os.getpid()}")
    cmd = [nvcc_path(), *NVCC_FLAGS, "-o", str(tmp), *map(str, SOURCES)]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build_library(force="--force" in sys.argv, verbose=True))
