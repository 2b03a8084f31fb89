"""Build libdilattn.so in-tree with nvcc for sm_100a.

    python -m sparse_long_sequence_dilated_b200.build [--ptxas-v]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "dilattn.cu")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdilattn.so")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(ptxas_verbose: bool = False, out: str = LIB) -> str:
    cmd = [
        nvcc_path(), "-O3", "-std=c++17",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-lineinfo", "-shared", "-Xcompiler", "-fPIC,-O3", "-cudart", "static",
        "-I", INCLUDE, "-I", os.path.join(PKG, "csrc"),
        "-o", out, SRC,
    ]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if ptxas_verbose:
        sys.stderr.write(res.stderr)
    return out


if __name__ == "__main__":
    build(ptxas_verbose="--ptxas-v" in sys.argv)
    print(LIB)
