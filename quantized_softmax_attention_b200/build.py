"""Build the kiattn CUDA library in-tree (sm_100a).

``python -m quantized_softmax_attention_b200.build`` compiles
``csrc/kiattn.cu`` into ``libkiattn.so`` next to this file with nvcc
(cross-compiles without a GPU).  No fast-math and no FMA contraction beyond
what the source spells out, so the weight stage's fp32 arithmetic is the
one written in ``csrc/kia_common.cuh``.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "kiattn.cu")
LIB = os.path.join(HERE, "libkiattn.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _sources():
    d = os.path.join(HERE, "csrc")
    out = [os.path.join(d, f) for f in os.listdir(d) if f.endswith((".cu", ".cuh"))]
    out.append(os.path.join(ROOT, "include", "kiattn.h"))
    return out


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(s) <= t for s in _sources()):
            return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++20", "--fmad=true", "-shared",
           "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"), "-o", tmp, SRC]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
    print(LIB)
