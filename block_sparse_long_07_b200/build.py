"""Build libmoba.so in-tree with nvcc for sm_100a.

    python -m block_sparse_long_07_b200.build [--force] [--verbose]
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmoba.so")
SOURCES = [os.path.join(CSRC, "moba_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(ROOT, "include", "moba.h")]


def nvcc_cmd(out, verbose=False):
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-o", out] + SOURCES
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in DEPS)


def build(force=False, verbose=False):
    if not force and not stale():
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.check_call(nvcc_cmd(tmp, verbose))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
