"""Build libfp8bl.so in-tree with nvcc for sm_100a.

    python -m fine_grained_block_token_b200.build [--verbose-ptxas]

The library is written next to this file so it travels with the source tree.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp8bl.so")
SOURCES = ["api.cu", "quant.cu", "gemm.cu", "gemm_pair.cu", "gemm_ue8m0.cu", "gemm_ue8m0_pair.cu", "gemm_rowwise.cu", "decode.cu", "fused.cu", "noalloc.cu"]
HEADERS = ["fp8bl_internal.h", "ptx_sm100.cuh", "quant_math.cuh"]
INCLUDE = os.path.join(os.path.dirname(HERE), "include", "fp8bl.h")


def nvcc() -> str:
    for cand in (os.environ.get("CUDA_HOME"), os.environ.get("CUDA_PATH")):
        if cand and os.path.exists(os.path.join(cand, "bin", "nvcc")):
            return os.path.join(cand, "bin", "nvcc")
    p = shutil.which("nvcc")
    if p:
        return p
    return "/usr/local/cuda/bin/nvcc"


def _inputs():
    srcs = [os.path.join(CSRC, s) for s in SOURCES if os.path.exists(os.path.join(CSRC, s))]
    return srcs, srcs + [os.path.join(CSRC, h) for h in HEADERS] + [INCLUDE, __file__]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _inputs()[1])


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not verbose_ptxas and up_to_date():
        return LIB
    srcs, _ = _inputs()
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared", "-o", tmp, *srcs]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose_ptxas:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
