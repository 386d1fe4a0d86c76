"""The library's host-side Hilbert order equals the pinned oracle order,
index for index (integer work: bit-exact)."""
import numpy as np
import pytest

import block_sparse_long_tiled_b200 as sk
from oracle.hilbert import hilbert_order


@pytest.mark.parametrize("grid", [(13, 32, 43, 17776), (13, 32, 43, 17888), (2, 3, 4, 24),
                                  (8, 8, 8, 512), (5, 7, 9, 300), (1, 1, 1, 1), (1, 1, 64, 64),
                                  (40, 3, 5, 599)])
def test_library_order_equals_oracle(grid):
    np.testing.assert_array_equal(sk.sskip_hilbert3d_order(*grid), hilbert_order(*grid))


def test_order_rejects_bad_arguments():
    for g in [(0, 1, 1, 1), (2, 2, 2, 9), (2, 2, 2, 0)]:
        with pytest.raises(sk.SSkipError):
            sk.sskip_hilbert3d_order(*g)
