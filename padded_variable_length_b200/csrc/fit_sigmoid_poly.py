"""Fits the polynomial g(e) ~ 1 / (1 + e) on e in [0, 1] that the kernels use for the
sigmoid (sm100.cuh, sigmoid_ex2): sigma(x) = g(e) for x >= 0 and e g(e) for x < 0, with
e = exp(-|x|) from the hardware exp2.  Minimises the maximum RELATIVE error (weights near
1/n are tiny, so relative, not absolute, error is what must stay below the bf16 rounding of
the weights) by Lawson's iteratively reweighted least squares, then reports the error of
the float32 Horner evaluation of the float32-rounded coefficients.

    python padded_variable_length_b200/csrc/fit_sigmoid_poly.py [degree]
"""
import sys

import numpy as np


def fit(deg: int, points: int = 20001, iters: int = 300):
    e = np.linspace(0.0, 1.0, points)
    g = 1.0 / (1.0 + e)
    V = np.vander(e, deg + 1, increasing=True)
    w = np.full(points, 1.0 / points)
    for _ in range(iters):
        W = np.sqrt(w) / g
        c, *_ = np.linalg.lstsq(V * W[:, None], g * W, rcond=None)
        r = np.abs(V @ c - g) / g
        w = w * r
        w /= w.sum()
    c32 = c.astype(np.float32)
    e32 = e.astype(np.float32)
    p = np.full_like(e32, c32[-1])
    for a in c32[-2::-1]:
        p = (p * e32 + a).astype(np.float32)
    rel32 = float(np.max(np.abs(p.astype(np.float64) - g) / g))
    return c32, rel32


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c, rel = fit(deg)
    print(f"degree {deg}: max relative error {rel:.3e} (2^{np.log2(rel):.2f})")
    for i, a in enumerate(c):
        print(f"  a{i} = {float(a):.9g}f")
