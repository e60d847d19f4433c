"""Builds libmagi_bca.so in-tree with nvcc for sm_100a.

Usage: python -m block_causal_attention_gqa_b200.build [--debug]
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmagi_bca.so")
SOURCES = ["bca_api.cu", "bca_fwd.cu", "bca_bwd.cu", "bca_bwd_split.cu", "bca_noalloc.cu", "bca_sched.cpp"]
DEPS = SOURCES + ["sm100.cuh", "bca_kernels.h", "bca_sched.h", "bca_norm.cuh", "bca_bwd_common.cuh"]


def nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def needs_build():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    paths = [os.path.join(CSRC, f) for f in DEPS] + [os.path.join(ROOT, "include", "magi_bca.h"), __file__]
    return any(os.path.getmtime(p) > t for p in paths if os.path.exists(p))


def build(force=False, verbose=False):
    if not force and not needs_build():
        return LIB
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-o", LIB]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
