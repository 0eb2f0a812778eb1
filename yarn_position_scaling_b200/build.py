"""Build libyarnattn.so in-tree (nvcc for sm_100a, static CUDA runtime).

    python -m yarn_position_scaling_b200.build [--force]

The library lands in ``yarn_position_scaling_b200/_build/libyarnattn.so``; the
binding in ``api.py`` loads it from there and raises if it is missing.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT_DIR = os.path.join(PKG, "_build")
LIB = os.path.join(OUT_DIR, "libyarnattn.so")
HEADER = os.path.join(ROOT, "include", "yarnattn.h")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh", ".cpp", ".h"))) + [HEADER]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in _sources() + [__file__])


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile (if stale) and return the path of libyarnattn.so."""
    if not force and not _stale():
        return LIB
    os.makedirs(OUT_DIR, exist_ok=True)
    objs = []
    common = ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include")]
    for src, extra in [("yarnattn.cu", ARCH + ["-lineinfo"]), ("rope_table.cpp", ARCH)]:
        obj = os.path.join(OUT_DIR, src + ".o")
        cmd = [NVCC] + common + extra + ["-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
