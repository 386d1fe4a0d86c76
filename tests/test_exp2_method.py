"""The FMA-pipe exp2 of the prefill kernel (exp2_fma2 in sm100_ptx.cuh),
evaluated step by step in float32 with the coefficients read from the header,
against float64 exp2: relative error within the stated 1.7e-4 over the range
the kernel feeds it, and -inf maps to (effectively) zero."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_long_tiled_b200", "csrc", "sm100_ptx.cuh")


def coefficients():
    src = open(HDR).read()
    body = src[src.index("exp2_fma2"):]
    vals = dict(re.findall(r"(kC\d) = ([0-9.eE+-]+)f", body))
    return [np.float32(vals[f"kC{i}"]) for i in range(4)]


def method(x, c):
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t + (-magic)).astype(np.float32)
    f = (n * np.float32(-1.0) + x).astype(np.float32)
    p = (c[3] * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    c = coefficients()
    x = np.concatenate([np.linspace(-126.0, 8.0, 1_000_001), np.linspace(-1, 1, 100_001)])
    x = x.astype(np.float32)
    got = method(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got - want) / want) < 1.7e-4


def test_integers_and_minus_infinity():
    c = coefficients()
    xs = np.arange(-20, 9, dtype=np.float32)
    got = method(xs, c)
    np.testing.assert_allclose(got, np.exp2(xs.astype(np.float64)), rtol=1e-4)
    assert method(np.float32(-np.inf), c) < 1e-37
