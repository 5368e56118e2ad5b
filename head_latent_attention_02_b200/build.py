"""Build libmla.so in-tree with nvcc for sm_100a (no GPU needed to compile)."""
from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libmla.so")
SOURCES = ["csrc/mla_lib.cu", "csrc/mla_static_ws.cu", "csrc/mla_append.cu",
           "csrc/mla_qknorm.cu", "csrc/mla_lowbit_tc.cu"]
DEPENDS = ["csrc/mla_lib.cu", "csrc/mla_static_ws.cu", "csrc/mla_append.cu", "csrc/mla_qknorm.cu",
           "csrc/mla_lowbit_tc.cu", "csrc/common.cuh",
           "csrc/ptx.cuh", "csrc/kernels_simt.cuh", "csrc/kernels_lowbit.cuh", "csrc/wgemm.cuh", "csrc/decode_tc.cuh", "../include/mla.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


def _nvcc() -> str:
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = os.path.join(home, "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(os.path.join(PKG, d)) > t for d in DEPENDS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libmla.so next to this file; returns its path."""
    if not force and not needs_build():
        return LIB
    cmd = [_nvcc(), *NVCC_FLAGS, "-I" + os.path.join(ROOT, "include"),
           "-I" + os.path.join(PKG, "csrc"), "-o", LIB + ".tmp",
           *[os.path.join(PKG, s) for s in SOURCES]]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stdout + res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
