"""Hilbert-curve token order for 3-D (T, H, W) token grids -- TEST
INFRASTRUCTURE ONLY (the library has its own implementation).

The SpargeAttn article ("Hilbert 曲线置换" under its technical details)
permutes the T x H x W visual tokens along a 3-D Hilbert curve before
flattening them to the L x d sequence, so that tokens adjacent in the
sequence are adjacent in space, which raises the similarity inside a block
and with it the share of blocks that can be skipped (its Table 4 compares
random, row-major, time-major and Hilbert orders).

Reading taken here for grids whose sides are not powers of two: each point
(t, h, w) gets the index of its position on the Hilbert curve of the smallest
2^b cube holding the grid, and the tokens are sorted by that index (points
outside the grid are simply absent). The index is computed with John
Skilling's transform ("Programming the Hilbert curve", AIP Conf. Proc. 707,
2004): coordinates -> "transposed" Hilbert index -> interleaved bits.
"""
from __future__ import annotations

import numpy as np


def hilbert_index(coords, bits: int) -> int:
    """Position of the point `coords` (n non-negative ints < 2^bits) along the
    n-dimensional Hilbert curve of side 2^bits."""
    x = [int(c) for c in coords]
    n = len(x)
    top = 1 << (bits - 1)
    # Undo the excess work of the curve's reflections and rotations, from the
    # coarsest bit down.
    q = top
    while q > 1:
        p = q - 1
        for i in range(n):
            if x[i] & q:
                x[0] ^= p
            else:
                t = (x[0] ^ x[i]) & p
                x[0] ^= t
                x[i] ^= t
        q >>= 1
    # Gray-encode.
    for i in range(1, n):
        x[i] ^= x[i - 1]
    t = 0
    q = top
    while q > 1:
        if x[n - 1] & q:
            t ^= q - 1
        q >>= 1
    for i in range(n):
        x[i] ^= t
    # Interleave the transposed form: bit j of every axis, from the top bit.
    h = 0
    for j in range(bits - 1, -1, -1):
        for i in range(n):
            h = (h << 1) | ((x[i] >> j) & 1)
    return h


def grid_bits(T: int, H: int, W: int) -> int:
    side = max(T, H, W)
    return max(1, int(np.ceil(np.log2(side))))


def raster_coords(T: int, H: int, W: int, L: int) -> np.ndarray:
    """(t, h, w) of the first L tokens of the t-major raster: [L, 3]."""
    i = np.arange(L)
    return np.stack([i // (H * W), (i // W) % H, i % W], axis=1)


def hilbert_order(T: int, H: int, W: int, L: int) -> np.ndarray:
    """perm [L] int32: perm[s] = raster index of the token placed at position s
    of the Hilbert-ordered sequence."""
    bits = grid_bits(T, H, W)
    xyz = raster_coords(T, H, W, L)
    keys = np.array([hilbert_index(p, bits) for p in xyz], dtype=np.int64)
    return np.argsort(keys, kind="stable").astype(np.int32)
