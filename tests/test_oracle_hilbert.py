"""Pins of the Hilbert-order oracle: the defining properties of a Hilbert
curve on full 2^b cubes (a bijection onto 0 .. 2^(n b) - 1 that starts at the
origin and moves by one unit step at a time), and a permutation of the tokens
on the video grid."""
import itertools

import numpy as np
import pytest

from oracle.hilbert import grid_bits, hilbert_index, hilbert_order, raster_coords


@pytest.mark.parametrize("n,bits", [(2, 1), (2, 3), (3, 1), (3, 2), (3, 3)])
def test_full_cube_is_a_unit_step_path_from_the_origin(n, bits):
    side = 1 << bits
    pts = list(itertools.product(range(side), repeat=n))
    idx = [hilbert_index(p, bits) for p in pts]
    assert sorted(idx) == list(range(side ** n))         # bijection
    path = [None] * side ** n
    for p, h in zip(pts, idx):
        path[h] = np.array(p)
    assert not path[0].any()                              # starts at the origin
    steps = [int(np.abs(path[i + 1] - path[i]).sum()) for i in range(len(path) - 1)]
    assert all(s == 1 for s in steps)                     # unit steps only


def test_coarse_structure_is_recursive():
    # The first 1/8 of a 3-D curve of side 8 fills one octant (side 4) entirely.
    bits = 3
    pts = list(itertools.product(range(8), repeat=3))
    first = [p for p in pts if hilbert_index(p, bits) < 64]
    lo = np.min(first, axis=0)
    hi = np.max(first, axis=0)
    assert np.all(hi - lo == 3) and np.all(lo % 4 == 0)


def test_video_grid_order_is_a_permutation_with_better_locality():
    T, H, W, L = 13, 32, 43, 17776
    assert grid_bits(T, H, W) == 6
    perm = hilbert_order(T, H, W, L)
    assert perm.dtype == np.int32 and np.array_equal(np.sort(perm), np.arange(L))
    xyz = raster_coords(T, H, W, L)
    # Tokens of one 128-token block sit in a smaller box than in raster order.
    def mean_extent(order):
        ext = []
        for s in range(0, L - 127, 128):
            p = xyz[order[s:s + 128]]
            ext.append(np.prod(p.max(0) - p.min(0) + 1))
        return np.mean(ext)
    assert mean_extent(perm) < 0.7 * mean_extent(np.arange(L))


def test_raster_coords():
    c = raster_coords(2, 3, 4, 24)
    assert tuple(c[0]) == (0, 0, 0) and tuple(c[5]) == (0, 1, 1) and tuple(c[23]) == (1, 2, 3)
