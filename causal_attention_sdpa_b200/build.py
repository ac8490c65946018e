"""Build libgpt_attn.so in-tree with nvcc for sm_100a.

Usage: python -m causal_attention_sdpa_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgpt_attn.so")
DEBUG_LIB = os.path.join(PKG, "libgpt_attn_debug.so")   # -DGPT_ATTN_DEBUG: bounds checks, load-skip hook
SOURCES = [os.path.join(CSRC, "gpt_attn.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + \
    [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def command(out: str, verbose: bool = False, debug: bool = False):
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I", CSRC, "-o", out] + SOURCES
    if debug:
        cmd.insert(1, "-DGPT_ATTN_DEBUG")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date(lib: str) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build the library (or, with debug=True, libgpt_attn_debug.so) if a source is newer."""
    lib = DEBUG_LIB if debug else LIB
    if force or not up_to_date(lib):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.run(command(tmp, verbose, debug), check=True)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    debug = "--debug" in sys.argv
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug=debug))
