"""Builds libnosa.so in-tree with nvcc for sm_100a (no JIT cache)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SO = os.path.join(HERE, "libnosa.so")
SRC = os.path.join(HERE, "csrc", "nosa_api.cu")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         "-Xcompiler", "-fPIC", "-shared", "-I" + os.path.join(ROOT, "include")]


def _inputs():
    return [SRC] + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + \
        [os.path.join(ROOT, "include", "nosa.h")]


def stale(so: str = SO) -> bool:
    if not os.path.exists(so):
        return True
    t = os.path.getmtime(so)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, extra=(), out: str = SO) -> str:
    if force or stale(out) or extra:
        cmd = [NVCC, *FLAGS, *extra, "-o", out, SRC]
        subprocess.check_call(cmd)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
