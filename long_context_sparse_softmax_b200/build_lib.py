"""Build liblc.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

Usage: python long_context_sparse_softmax_b200/build_lib.py [--force] [--ptxas-v]
(run by path: importing the package itself needs the built library)
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "liblc.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["lc_abi.cu", "k_prep.cu", "k_index.cu", "k_topk.cu", "k_attn.cu", "k_attn_combine.cu", "k_index_tc.cu", "k_attn_tc.cu", "k_attn_tc8.cu", "k_quant.cu", "k_outproj.cu", "lc_noalloc.cu"]
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-O3",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return [os.path.join(CSRC, s) for s in SOURCES]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    deps.append(os.path.join(ROOT, "include", "lc.h"))
    return all(os.path.getmtime(d) <= t for d in deps)


def build(verbose: bool = False, force: bool = False, extra=()) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [NVCC, *FLAGS, *extra, *sources(), "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(verbose=True, force="--force" in sys.argv,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
