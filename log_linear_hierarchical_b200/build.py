"""Builds libllsa.so (the CUDA C-ABI library) in-tree for sm_100a with nvcc.

Usage: python -m log_linear_hierarchical_b200.build [--verbose-ptxas] [--define NAME=VALUE ...]

--define passes a compile-time switch to nvcc, e.g. LLSA_KV_STAGES=3 for a deeper dK/dV ring.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libllsa.so")
SOURCES = ["llsa_api.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources_newer_than_lib() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "llsa.h")]
    return any(os.path.getmtime(f) > t for f in files if os.path.isfile(f))


def build(force: bool = False, ptxas_verbose: bool = False, defines: tuple[str, ...] = ()) -> str:
    if not force and not sources_newer_than_lib():
        return LIB
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-I", os.path.join(ROOT, "include"), "-o", LIB + ".tmp"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-D" + d for d in defines]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if ptxas_verbose:
        sys.stderr.write(res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    args = sys.argv[1:]
    defs = tuple(args[i + 1] for i, a in enumerate(args) if a == "--define" and i + 1 < len(args))
    build(force=True, ptxas_verbose="--verbose-ptxas" in args, defines=defs)
    print(LIB)
