"""Build libbitlinear.so in-tree with nvcc for sm_100a (B200).

Usage: python -m ternary_weight_linear_absmax_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libbitlinear.so")
SOURCES = [os.path.join(CSRC, "bitlinear.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(INCLUDE, "bitlinear.h")]

# Host table-lookup library (x86-64; instruction set chosen at run time).
CPU_SRC = os.path.join(PKG, "cpu", "lut_gemm.cpp")
CPU_LIB = os.path.join(PKG, "libbitlinear_lut_cpu.so")
CPU_DEPS = [CPU_SRC, os.path.join(INCLUDE, "bitlinear_lut_cpu.h")]
CXX_FLAGS = ["-O3", "-std=c++17", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
             "-shared", "-fPIC"]

NVCC_FLAGS = [
    "-std=c++17", "-O3",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build_cpu(force: bool = False, verbose: bool = False) -> str:
    """Compile the host table-lookup library with g++."""
    if (not force and os.path.exists(CPU_LIB)
            and all(os.path.getmtime(d) <= os.path.getmtime(CPU_LIB) for d in CPU_DEPS)):
        return CPU_LIB
    tmp = CPU_LIB + f".tmp{os.getpid()}"
    cmd = ["g++", *CXX_FLAGS, "-I", INCLUDE, CPU_SRC, "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, CPU_LIB)
    return CPU_LIB


def build(force: bool = False, verbose: bool = False) -> str:
    build_cpu(force, verbose)
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, *SOURCES, "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
