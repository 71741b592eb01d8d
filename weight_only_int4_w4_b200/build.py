"""Build libw4.so in-tree with nvcc for sm_100a (B200)."""
from __future__ import annotations

import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
MAIN = os.path.join(SRC_DIR, "libw4.cu")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libw4.so")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    out = [os.path.join(INCLUDE, "w4.h")]
    for f in os.listdir(SRC_DIR):
        if f.endswith((".cu", ".cuh")):
            out.append(os.path.join(SRC_DIR, f))
    return out


def build_library(force: bool = False, verbose: bool = False) -> str:
    """Compile every kernel of the library (one translation unit) into libw4.so."""
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in _sources())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cmd = [nvcc_path(), "-O3", "-std=c++17",
           "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", "-I" + INCLUDE,
           "-o", LIB + ".tmp", MAIN]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build_library(force=True))
