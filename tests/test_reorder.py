"""Token permutations from the C library against the oracle's reading (host
logic, no GPU)."""
import numpy as np
import pytest

import block_sparse_attention_14_b200 as bsa
from oracle import bsa_oracle as O


@pytest.mark.parametrize("mode", ["raster", "cube", "morton"])
@pytest.mark.parametrize("grid", [(21, 45, 80, 0), (13, 30, 45, 226), (33, 45, 80, 0), (1, 2, 8, 0), (5, 9, 6, 3)])
def test_library_permutation_equals_oracle(mode, grid):
    T, Hg, Wg, text = grid
    assert np.array_equal(bsa.token_permutation(T, Hg, Wg, text, mode).numpy(),
                          O.token_permutation(T, Hg, Wg, text, mode))


def test_permutation_rejects_bad_arguments():
    L = bsa.lib()
    import ctypes

    buf = (ctypes.c_int32 * 16)()
    assert L.bsa_token_permutation(0, 2, 8, 0, 1, buf) == 1
    assert L.bsa_token_permutation(1, 2, 8, 0, 3, buf) == 1
    assert L.bsa_token_permutation(1, 2, 8, -1, 1, buf) == 1
    assert L.bsa_token_permutation(1, 2, 8, 0, 1, None) == 1
    s = bsa.Shape(1, 1, 16, 12)
    assert L.bsa_permute_tokens(256, 512, s, 1024, 0, None) == 1      # d not a multiple of 8
    assert L.bsa_permute_tokens(256, 256, bsa.Shape(1, 1, 16, 64), 1024, 0, None) == 1  # src == dst
