"""Builds libmagi_bca.so in-tree with nvcc for sm_100a.

Usage: python -m block_causal_attention_gqa_b200.build [-v] [--debug]

--debug builds libmagi_bca_debug.so instead, with -DMAGI_BCA_DEBUG: every
attention kernel checks its work unit against the problem's sizes and, if a
unit is out of range, records a device status code (read as
MAGI_BCA_DEVICE_CHECK) and returns before touching memory.  The binding loads
it when MAGI_BCA_LIBRARY names its path.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmagi_bca.so")
DEBUG_LIB = os.path.join(HERE, "libmagi_bca_debug.so")
SOURCES = ["bca_api.cu", "bca_fwd.cu", "bca_bwd.cu", "bca_bwd_split.cu", "bca_noalloc.cu", "bca_sched.cpp"]
DEPS = SOURCES + ["sm100.cuh", "bca_kernels.h", "bca_sched.h", "bca_norm.cuh", "bca_bwd_common.cuh", "bca_mask.cuh"]


def nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def needs_build(lib=LIB):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    paths = [os.path.join(CSRC, f) for f in DEPS] + [os.path.join(ROOT, "include", "magi_bca.h"), __file__]
    return any(os.path.getmtime(p) > t for p in paths if os.path.exists(p))


def build(force=False, verbose=False, debug=False):
    lib = DEBUG_LIB if debug else LIB
    if not force and not needs_build(lib):
        return lib
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-o", lib]
    if debug:
        cmd += ["-DMAGI_BCA_DEBUG"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
