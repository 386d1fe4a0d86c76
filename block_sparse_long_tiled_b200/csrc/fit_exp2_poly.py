"""Fits the polynomial p(f) ~ 2**f on f in [-1/2, 1/2] used by the prefill
kernel's FMA-pipe exp2 (exp2_fma in sm100_ptx.cuh), minimising the maximum
relative error by iteratively reweighted least squares (a Lawson iteration
toward the minimax fit) on a dense grid, then reports the error of the whole
method in float32: x = n + f with n = round(x) by adding 1.5 * 2**23,
2**x = p(f) * 2**n with the exponent added to the bits of p(f).

    python fit_exp2_poly.py [degree]
"""
import sys

import numpy as np


def fit(degree: int, iters: int = 200):
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones_like(f)
    for _ in range(iters):
        W = w / y  # relative error weighting
        c, *_ = np.linalg.lstsq(V * W[:, None], y * W, rcond=None)
        err = np.abs(V @ c - y) / y
        w = w * (err + 1e-30)
        w /= w.sum()
    return c, float(np.max(np.abs(V @ c - y) / y))


def emulate(x, c):
    """The kernel's method in float32 (clamped at -126)."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.float32(c[-1])
    for ci in c[-2::-1]:
        p = (p * f + np.float32(ci)).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = fit(deg)
    c32 = c.astype(np.float32)
    x = np.linspace(-126.0, 8.0, 2_000_001).astype(np.float32)
    got = emulate(x, c32).astype(np.float64)
    rel = np.abs(got - np.exp2(x.astype(np.float64))) / np.exp2(x.astype(np.float64))
    print("degree", deg, "fit max rel err", e)
    print("coefficients (c0..c%d):" % deg, ", ".join(repr(float(v)) + "f" for v in c32))
    print("method max rel err over [-126, 8]:", rel.max())
