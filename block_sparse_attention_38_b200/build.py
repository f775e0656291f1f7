"""Build the C-ABI shared library libbsa.so in-tree with nvcc for sm_100a.

    python -m block_sparse_attention_38_b200.build [--force] [--verbose-ptxas]

The library holds the host pattern builder (bsa_pattern.cpp) and four CUDA
translation units: the forward launcher with its kernel (bsa_forward.cu),
top-k block selection (bsa_topk.cu), the decode step (bsa_decode.cu) and
the backward pass (bsa_backward.cu).  CUDA runtime is linked
statically; the driver's tensor-map encoder is looked up at run time, so the
library loads on a machine without a GPU (only compute calls need one).
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = [os.path.join(CSRC, "bsa_pattern.cpp"), os.path.join(CSRC, "bsa_forward.cu"),
           os.path.join(CSRC, "bsa_topk.cu"), os.path.join(CSRC, "bsa_decode.cu"),
           os.path.join(CSRC, "bsa_backward.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith(".cuh")] + [
    os.path.join(ROOT, "include", "bsa.h")]
LIB = os.path.join(HERE, "libbsa.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-I" + os.path.join(ROOT, "include"),
]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if verbose_ptxas else []) + SOURCES + ["-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    args = ap.parse_args(argv)
    print(build(force=args.force, verbose_ptxas=args.verbose_ptxas))


if __name__ == "__main__":
    sys.exit(main())
