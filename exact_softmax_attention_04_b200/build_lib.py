"""Compile the CUDA library libattn_b200.so in-tree for sm_100a.

Usage: python -m exact_softmax_attention_04_b200.build_lib [--force] [--verbose]
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libattn_b200.so")
SOURCES = [os.path.join(CSRC, f) for f in ("attn_api.cu", "attn_bwd_api.cu", "attn_decode_api.cu")]
HEADERS = [os.path.join(CSRC, f) for f in ("attn_fwd_kernel.cuh", "attn_bwd_kernel.cuh",
                                            "attn_bwd_fused_kernel.cuh", "attn_decode_kernel.cuh", "sm100.cuh",
                                            "attn_host.h")] + [
    os.path.join(ROOT, "include", "attn.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-shared",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [_nvcc()] + NVCC_FLAGS + ["-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", tmp] + SOURCES
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


def build_variant(out_path: str, defines) -> str:
    """Build the same sources with extra preprocessor definitions into
    ``out_path`` (used by the fault-injection test; never the library)."""
    cmd = [_nvcc()] + NVCC_FLAGS + ["-I", os.path.join(ROOT, "include"), "-I", CSRC]
    cmd += [f"-D{d}" for d in defines]
    cmd += ["-o", str(out_path)] + SOURCES
    subprocess.check_call(cmd)
    return str(out_path)


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose, verbose=a.verbose), file=sys.stderr)
