"""Fits the degree-3 polynomial for 2^f on f in [-1/2, 1/2] used by exp2_fma2 in
device_common.cuh (part of the softmax exponentials run on the FMA pipe instead of the MUFU).

Method: least squares on 4000 Chebyshev nodes with weights 1/2^f (relative error), then
Lawson's iteration, which reweights toward the minimax (equal-ripple) solution.  Prints the
float32 coefficients and the maximum relative error of their float32 evaluation.

    python head_wise_sparse_b200/csrc/exp2_poly_fit.py
"""
import numpy as np


def fit(deg: int = 3, nodes: int = 4000, iters: int = 200):
    f = np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes) * 0.5
    y = np.exp2(f)
    A = np.vstack([f ** k for k in range(deg + 1)]).T
    w = np.ones_like(f)
    for _ in range(iters):
        W = w / y
        c, *_ = np.linalg.lstsq(A * W[:, None], y * W, rcond=None)
        e = np.abs(A @ c - y) / y
        w = w * np.sqrt(e / e.max()) + 1e-12
        w /= w.mean()
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(c32[::-1], g.astype(np.float32)).astype(np.float64)
    return c32, float(np.max(np.abs(p - np.exp2(g)) / np.exp2(g)))


if __name__ == "__main__":
    c, err = fit()
    print("coefficients (c0..c3):", ", ".join(f"{x:.11f}f" for x in c))
    print(f"max relative error (float32 evaluation): {err:.3e}")
