"""Build libnabla.so in-tree with nvcc for sm_100a.

Usage: python -m block_sparse_attention_flatten_b200.build [--force] [--verbose-ptxas]

The library links the CUDA runtime statically and resolves the driver's
tensor-map encoder at run time, so it loads on a machine without a GPU
driver (the compute calls then fail with NABLA_ERR_CUDA).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libnabla.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def nvcc_cmd(out: str, ptxas_verbose: bool = False):
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-o", out, os.path.join(CSRC, "nabla_api.cu")]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    newest = max(os.path.getmtime(p) for p in sources())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest and not ptxas_verbose:
        return LIB
    tmp = LIB + ".tmp"
    subprocess.check_call(nvcc_cmd(tmp, ptxas_verbose))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
