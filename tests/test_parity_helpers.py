"""The near-tie selection check of the GPU parity helpers, on the CPU.

valid_selection decides whether a GPU selection that differs from the
oracle's at a near-tie is still a correct one.  It must accept the oracle's
own selections and swaps inside the 1e-4 band, and reject everything else: a
clearly worse block kept, a clearly better one dropped, a missing own block, a
wrong count, a future block.
"""
import numpy as np

from oracle import moba_ref as R
from tests.parity import valid_selection


def test_oracle_selection_is_valid():
    rng = np.random.default_rng(3)
    for _ in range(300):
        j = int(rng.integers(0, 60))
        topk = int(rng.integers(1, 14))
        sc = rng.standard_normal(j).astype(np.float32)
        sel, _ = R.select_blocks(sc, j, topk)
        assert valid_selection(sc, j, topk, sel)


def test_swap_inside_band_is_valid_outside_is_not():
    j, topk = 10, 4
    sc = np.array([5.0, 4.0, 3.0, 2.0, 1.99995, 1.0, 0.5, 0.0, -1.0, -2.0], dtype=np.float32)
    ref, tie = R.select_blocks(sc, j, topk)
    assert ref == [0, 1, 2, 10] and not tie
    sc2 = sc.copy()
    sc2[3] = 3.0 - 1e-5          # blocks 2 and 3 now within the band
    ref2, tie2 = R.select_blocks(sc2, j, topk)
    assert tie2
    assert valid_selection(sc2, j, topk, [0, 1, 3, 10])   # swapped inside the band
    assert valid_selection(sc2, j, topk, [0, 1, 2, 10])
    assert not valid_selection(sc2, j, topk, [0, 1, 4, 10])   # clearly worse block kept
    assert not valid_selection(sc2, j, topk, [1, 2, 3, 10])   # clearly better block dropped


def test_malformed_selections_are_rejected():
    sc = np.arange(8, dtype=np.float32)[::-1].copy()     # block 0 best
    j, topk = 8, 3
    assert valid_selection(sc, j, topk, [0, 1, 8])
    assert not valid_selection(sc, j, topk, [0, 1])        # own block missing
    assert not valid_selection(sc, j, topk, [0, 8])        # too few past blocks
    assert not valid_selection(sc, j, topk, [0, 1, 2, 8])  # too many
    assert not valid_selection(sc, j, topk, [0, 0, 8])     # repeated block
    assert not valid_selection(sc, j, topk, [0, 1, 9])     # future block
    # every block 0..j when j + 1 <= topk
    assert valid_selection(sc[:2], 2, 3, [0, 1, 2])
    assert not valid_selection(sc[:2], 2, 3, [0, 2])
