"""Compile libsbfa.so (the C-ABI library) for sm_100a, in-tree.

Usage: python block_sparse_flashattention_sbfa_b200/build.py [--verbose-ptxas]
(run it as a script: importing the package needs the library it builds).
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libsbfa.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh")))


def build(verbose_ptxas=False, force=False):
    srcs = sources() + [os.path.join(ROOT, "include", "sbfa.h")]
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(s) for s in srcs)):
        return LIB
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "--cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-o", LIB + ".tmp", os.path.join(CSRC, "sbfa_api.cu")]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose_ptxas="--verbose-ptxas" in sys.argv, force=True))
