"""Build the library (liblpfa.so) in-tree with nvcc for sm_100a.

Usage: ``python precision_attention_forward_b200/build.py [--verbose]`` (run as a file: importing
the package loads the library being built). The shared library links the CUDA runtime
statically and needs only the driver at run time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG_DIR, "liblpfa.so")

SOURCES = ["lpfa.cu"]
HEADERS = ["ptx.cuh", "quantize.cuh", "attn_fwd.cuh", "attn_fwd_pp.cuh", "attn_bwd.cuh", "dequantize.cuh"]


def nvcc_path() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def nvcc_flags(ptxas_verbose: bool = False):
    flags = [
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
        "-I", INCLUDE, "-I", CSRC,
        "--expt-relaxed-constexpr",
    ]
    if ptxas_verbose:
        flags += ["-Xptxas", "-v"]
    return flags


def needs_rebuild() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "lpfa.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_rebuild():
        return LIB_PATH
    cmd = [nvcc_path()] + nvcc_flags(verbose) + [
        "-shared", "-cudart", "static",
        "-o", LIB_PATH + ".tmp",
    ] + [os.path.join(CSRC, s) for s in SOURCES] + ["-ldl", "-lpthread", "-lrt"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed building liblpfa.so")
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB_PATH)
