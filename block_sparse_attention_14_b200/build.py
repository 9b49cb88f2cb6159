"""Builds libbsa.so (the C-ABI library) in-tree for sm_100a with nvcc.

Usage: python -m block_sparse_attention_14_b200.build [--verbose]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libbsa.so")
SOURCES = ["bsa_api.cu", "bsa_select.cu", "bsa_dots_tc.cu", "bsa_attn.cu", "bsa_noalloc.cu", "bsa_reorder.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def build(verbose: bool = False, extra: list[str] | None = None, out: str = LIB) -> str:
    """Compile every CUDA source into one shared library; returns its path."""
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    cmd = [nvcc(), "-shared", "-Xcompiler", "-fPIC", "-O3", "-lineinfo", "-std=c++17",
           *ARCH, "-I", INCLUDE, "-I", CSRC, "-o", out, *srcs]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if extra:
        cmd[1:1] = extra
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    return out


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv))
