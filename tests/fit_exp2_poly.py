"""Fits the polynomial the kernels use for part of their exp2 work.

2^x is split as 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]; 2^f
is approximated by a cubic fitted here by the Remez exchange algorithm
(minimax relative error).  The kernel offloads one exponential in four to
this polynomial on the FMA pipe, so the MUFU unit is not the bottleneck of
the softmax.  The result feeds a bf16 operand (rounding 2^-9), and the cubic's
maximum relative error is ~7.5e-5.

    python tests/fit_exp2_poly.py
prints the coefficients (fp32) that exp2_poly_pair in
block_causal_attention_gqa_b200/csrc/sm100.cuh uses, and their errors;
tests/test_exp2_poly.py re-runs the fit and checks those constants.
"""
import numpy as np


def remez(degree, a=-0.5, b=0.5, iters=40):
    n_pts = degree + 2
    x = np.sort(0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n_pts) / (n_pts - 1)))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        m = np.zeros((n_pts, n_pts))
        for i in range(n_pts):
            m[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            m[i, degree + 1] = (-1) ** i * np.exp2(x[i])
        coef = np.linalg.solve(m, np.exp2(x))[:degree + 1]
        err = (np.polyval(coef[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        turn = [0] + [i for i in range(1, len(grid) - 1)
                      if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [len(grid) - 1]
        sel = [turn[0]]
        for i in turn[1:]:
            if np.sign(err[i]) != np.sign(err[sel[-1]]):
                sel.append(i)
            elif abs(err[i]) > abs(err[sel[-1]]):
                sel[-1] = i
        if len(sel) >= n_pts:
            sel = sorted(sorted(sel, key=lambda i: -abs(err[i]))[:n_pts])
            x = grid[sel]
    return coef, float(np.max(np.abs(err)))


def fp32_error(coef):
    c = np.asarray(coef, dtype=np.float32)
    t = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = np.float32(c[-1]) * np.ones_like(t)
    for k in range(len(c) - 2, -1, -1):
        p = p * t + c[k]
    ref = np.exp2(t.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


if __name__ == "__main__":
    coef, err = remez(3)
    print("coefficients c0..c3 (fp32):", [float(np.float32(v)) for v in coef])
    print(f"minimax relative error {err:.3e}; evaluated in fp32 {fp32_error(coef):.3e}")
