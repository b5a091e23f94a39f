"""Fits the polynomials the GEMM epilogue uses for GELU's tail probability.

The epilogue computes GELU(x) = x Phi(x) as max(x, 0) - a q with a = min(|x|, 6) and
q = Phi(-a), the standard normal tail (for |x| <= 6 that is exact algebra; beyond, q is
below 1e-9 and the product below 6e-9), and takes q = 2^g(a), g a polynomial in a that
approximates log2 Phi(-a) on [0, 6].  There are two fits, one per type of C:

- fp32 C: degree 6, the error in g weighted by d GELU / d g = a Phi(-a) ln 2, so an error
  in g counts for what it costs in GELU;
- fp16 C: degree 5, the same weight divided by the fp16 unit in the last place of
  a Phi(-a), so the error counts in units of the fp16 result (for x < 0 the result is
  -a Phi(-a); for x > 0 it is larger and the relative error smaller).

Both are made near-minimax by Lawson's iteratively reweighted least squares; the
reference values come from scipy.special.log_ndtr.  Run it to print the coefficients
(float32, lowest degree first) and the errors they give, evaluated in float32 the way
the kernel does (Horner with fused multiply-adds, exact exp2 in place of the
hardware's): the fp32 fit's largest GELU error on [-8, 8], and the fp16 fit's largest
error in fp16 units in the last place over every fp16 input in [-16, 16].

    python fit_gelu_tail.py
"""

import numpy as np
from scipy.special import log_ndtr, ndtr

A_MAX = 6.0
DEGREE = {"f32": 6, "f16": 5}


def ulp_f16(v: np.ndarray) -> np.ndarray:
    """The fp16 unit in the last place at |v| (subnormal spacing below 2^-14)."""
    e = np.floor(np.log2(np.maximum(np.abs(v).astype(np.float64), 2.0 ** -14)))
    return 2.0 ** (e - 10)


def fit(out: str, a_max: float = A_MAX, iters: int = 60) -> np.ndarray:
    degree = DEGREE[out]
    a = np.linspace(0.0, a_max, 60001)
    g = log_ndtr(-a) / np.log(2.0)
    w = np.maximum(a * ndtr(-a) * np.log(2.0), 1e-12)
    if out == "f16":
        w = np.maximum(w / ulp_f16(a * ndtr(-a)), 1e-6)
        iters = 80
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
    c32, c16 = fit("f32"), fit("f16")
    print("fp32 C coefficients:", ", ".join(f"{float(c):.9g}f" for c in c32))
    x = np.linspace(-8, 8, 640001).astype(np.float32)
    ref = x.astype(np.float64) * ndtr(x.astype(np.float64))
    print(f"  max |GELU error| on [-8, 8]: {np.abs(gelu_f32(x, c32) - ref).max():.3g}")
    print("fp16 C coefficients:", ", ".join(f"{float(c):.9g}f" for c in c16))
    h = np.arange(0, 65536, dtype=np.uint16).view(np.float16)
    h = h[np.isfinite(h) & (np.abs(h) <= 16)].astype(np.float32)
    ref = h.astype(np.float64) * ndtr(h.astype(np.float64))
    print(f"  max GELU error in fp16 units in the last place (every fp16 input in [-16, 16]): "
          f"{(np.abs(gelu_f32(h, c16) - ref) / ulp_f16(ref)).max():.3g}")
