"""Fits the polynomial the GEMM epilogue uses for GELU's tail probability.

The epilogue computes GELU(x) = x Phi(x) as max(x, 0) - a q with a = min(|x|, 6) and
q = Phi(-a), the standard normal tail (for |x| <= 6 that is exact algebra; beyond, q is
below 1e-9 and the product below 6e-9), and takes q = 2^g(a), g a polynomial in a of
degree 6 that approximates log2 Phi(-a) on [0, 6].  The fit weights the error in g by
d GELU / d g = a Phi(-a) ln 2 (so an error in g costs what it costs in GELU) and is made
near-minimax by Lawson's iteratively reweighted least squares.  The reference values
come from scipy.special.log_ndtr.  Run it to print the coefficients (float32, lowest
degree first) and the GELU error they give, evaluated in float32 the way the kernel
does (Horner with fused multiply-adds, exact exp2 in place of the hardware's).

    python fit_gelu_tail.py
"""

import numpy as np
from scipy.special import log_ndtr, ndtr

A_MAX = 6.0
DEGREE = 6


def fit(degree: int = DEGREE, a_max: float = A_MAX, iters: int = 60) -> np.ndarray:
    a = np.linspace(0.0, a_max, 60001)
    g = log_ndtr(-a) / np.log(2.0)
    w = np.maximum(a * ndtr(-a) * np.log(2.0), 1e-12)
    V = np.vander(a / a_max, degree + 1, increasing=True)
    lw = np.ones_like(a)
    for _ in range(iters):
        sw = np.sqrt(lw) * w
        c, *_ = np.linalg.lstsq(V * sw[:, None], g * sw, rcond=None)
        e = np.abs(V @ c - g) * w
        lw = lw * e
        lw /= lw.sum()
    return (c / a_max ** np.arange(degree + 1)).astype(np.float32)


def gelu_f32(x: np.ndarray, coef: np.ndarray, a_max: float = A_MAX) -> np.ndarray:
    x = x.astype(np.float32)
    a = np.minimum(np.abs(x), np.float32(a_max))
    g = np.full_like(a, coef[-1])
    for c in coef[-2::-1]:
        g = (g.astype(np.float64) * a + np.float64(c)).astype(np.float32)
    q = np.exp2(g.astype(np.float64)).astype(np.float32)
    return (np.maximum(x, 0).astype(np.float64) - a.astype(np.float64) * q).astype(np.float32)


if __name__ == "__main__":
    coef = fit()
    print("coefficients:", ", ".join(f"{float(c):.9g}f" for c in coef))
    x = np.linspace(-8, 8, 640001).astype(np.float32)
    ref = x.astype(np.float64) * ndtr(x.astype(np.float64))
    print(f"max |GELU error| on [-8, 8]: {np.abs(gelu_f32(x, coef) - ref).max():.3g}")
