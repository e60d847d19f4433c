"""The cubic that computes part of the kernels' exponentials (exp2_poly_pair in
block_causal_attention_gqa_b200/csrc/sm100.cuh).

CPU: re-runs the Remez fit (tests/fit_exp2_poly.py) and checks that the
constants in the source are that fit rounded to fp32, and that the cubic's
relative error on [-1/2, 1/2], evaluated in fp32, stays within 7.6e-5.
GPU: the device function against CUDA's exp2f over [-125, 8.5] (the range
the kernels feed it), through a small test kernel compiled here."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from tests import fit_exp2_poly as fit

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SM100 = os.path.join(ROOT, "block_causal_attention_gqa_b200", "csrc", "sm100.cuh")
BOUND = 7.6e-5


def source_coefficients():
    """c3, c2, c1, c0 as written in exp2_poly_pair (Horner order)."""
    src = open(SM100).read()
    body = src[src.index("void exp2_poly_pair"):]
    body = body[:body.index("\n}\n")]
    # the polynomial's constants are the pairs after the rounding step's (-1, -1)
    vals = [float(v) for v in re.findall(r"f2_pack\(([-0-9.e]+)f, \1f\)", body)]
    return [v for v in vals if v != -1.0]


def test_source_constants_are_the_remez_fit():
    coef, err = fit.remez(3)
    c = [float(np.float32(v)) for v in coef]              # c0..c3
    src = source_coefficients()
    assert len(src) == 4, src
    want = [c[3], c[2], c[1], c[0]]
    for got, w in zip(src, want):
        assert abs(got - w) <= 4 * np.spacing(np.float32(abs(w))), (src, want)
    assert err <= 7.5e-5
    assert fit.fp32_error(coef) <= BOUND


def _build_probe():
    out_dir = os.path.join(HERE, "_build")
    os.makedirs(out_dir, exist_ok=True)
    so = os.path.join(out_dir, "exp2_poly_probe.so")
    src = os.path.join(HERE, "exp2_poly_probe.cu")
    if not os.path.exists(so) or os.path.getmtime(so) < max(os.path.getmtime(src), os.path.getmtime(SM100)):
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-shared",
                        "-Xcompiler", "-fPIC", "-o", so, src], check=True)
    return so


@pytest.mark.gpu
def test_exp2_poly_pair_against_exp2f_on_the_kernels_range():
    import torch
    lib = ctypes.CDLL(_build_probe())
    lib.exp2_poly_probe.restype = ctypes.c_int
    n = 1 << 22
    x = torch.linspace(-125.0, 8.5, n, device="cuda", dtype=torch.float32)
    # also every value near the rounding boundaries j +- 1/2 of the split
    half = torch.arange(-125, 9, device="cuda", dtype=torch.float32) + 0.5
    x = torch.cat([x, half, half - 1e-6, half + 1e-6]).clamp(-125.0, 8.5).contiguous()
    poly = torch.empty_like(x)
    ref = torch.empty_like(x)
    st = lib.exp2_poly_probe(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(poly.data_ptr()),
                             ctypes.c_void_p(ref.data_ptr()), ctypes.c_int(x.numel()))
    assert st == 0
    torch.cuda.synchronize()
    rel = ((poly.double() - ref.double()).abs() / ref.double()).max().item()
    print(f"exp2_poly_pair vs exp2f on [-125, 8.5]: max relative error {rel:.3e}")
    assert rel <= BOUND
