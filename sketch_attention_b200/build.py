"""Builds libsketchattn.so in-tree with nvcc for sm_100a.

    python -m sketch_attention_b200.build [--debug]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsketchattn.so")
SOURCES = ["api.cu", "gemm.cu", "sa_simt.cu", "sa_tc.cu", "sa_bwd_tc.cu", "sa_refine.cu", "sa_refine_bwd.cu", "sa_tokenwise.cu", "sa_noalloc.cu", "stca.cu",
           "stca_tc.cu", "stca_full.cu", "stca_ffn_tc.cu", "stca_bwd.cu", "events.cu", "measure.cu", "tc_gemm.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def sources():
    return [os.path.join(CSRC, s) for s in SOURCES]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")]
    deps.append(os.path.join(HERE, "..", "include", "sketch_attn.h"))
    return all(os.path.getmtime(p) <= t for p in deps if os.path.exists(p))


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "--expt-relaxed-constexpr", "-I" + os.path.join(HERE, "..", "include"),
           *extra, "-o", LIB + ".tmp", *sources(), "-lcuda"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    args = sys.argv[1:]
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in args else []
    build(force=True, verbose=True, extra=extra)
    print(LIB)
