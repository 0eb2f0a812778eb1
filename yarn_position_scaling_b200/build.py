"""Build libyarnattn.so in-tree (nvcc for sm_100a, static CUDA runtime).

    python -m yarn_position_scaling_b200.build [--force]

The library lands in ``yarn_position_scaling_b200/_build/libyarnattn.so``; the
binding in ``api.py`` loads it from there and raises if it is missing.  A second
build of the same sources with the failure-path test hook compiled in
(``-DYR_FAULT_HOOKS``) lands beside it as ``libyarnattn_faulthooks.so``; only the
failure-detection test loads that one.
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
LIB_FAULT_HOOKS = os.path.join(OUT_DIR, "libyarnattn_faulthooks.so")
HEADER = os.path.join(ROOT, "include", "yarnattn.h")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh", ".cpp", ".h"))) + [HEADER]


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in _sources() + [__file__])


def build(force: bool = False, verbose: bool = False, fault_hooks: bool = False) -> str:
    """Compile (if stale) and return the path of libyarnattn.so, or with fault_hooks=True
    of the test build libyarnattn_faulthooks.so."""
    lib = LIB_FAULT_HOOKS if fault_hooks else LIB
    if not force and not _stale(lib):
        return lib
    os.makedirs(OUT_DIR, exist_ok=True)
    tag = ".fh" if fault_hooks else ""
    objs = []
    common = ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include")]
    if fault_hooks:
        common += ["-DYR_FAULT_HOOKS"]
    for src, extra in [("yarnattn.cu", ARCH + ["-lineinfo"]), ("rope_table.cpp", ARCH),
                       ("host_prefill.cpp", ARCH)]:
        obj = os.path.join(OUT_DIR, src + tag + ".o")
        cmd = [NVCC] + common + extra + ["-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
    print(build(force="--force" in sys.argv, verbose=True, fault_hooks=True))
