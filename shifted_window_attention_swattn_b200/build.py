"""Builds libbasa_swattn.so in-tree with nvcc for sm_100a.

    python -m shifted_window_attention_swattn_b200.build [--force]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = [os.path.join(HERE, "csrc", "swattn_sm100.cu")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", "ptx_sm100.cuh"),
                  os.path.join(HERE, "csrc", "softmax_sm100.cuh"),
                  os.path.join(ROOT, "include", "basa_swattn.h")]
LIB = os.path.join(HERE, "libbasa_swattn.so")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str) -> list:
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
            "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
            "-o", out] + SOURCES


def build(force: bool = False, verbose: bool = False) -> str:
    fresh = os.path.exists(LIB) and all(
        os.path.getmtime(LIB) >= os.path.getmtime(p) for p in DEPS)
    if fresh and not force:
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = command(tmp)
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
