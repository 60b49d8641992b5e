"""The index-mismatch report of the GPU tests (CPU only)."""
import numpy as np

from _ties import index_mismatch, selection_gap


def test_selection_gap():
    gap, scale = selection_gap(np.array([0.5, 3.0, -2.0, 2.5]), 2)
    assert gap == 2.0 and scale == 3.0
    assert selection_gap(np.array([1.0, 2.0]), 2) == (None, None)


def test_near_tie_label():
    l = np.array([1.0, 4.0, 4.0 - 1e-15, 0.0])
    assert "a near tie" in index_mismatch("t", [2], [1], l)
    assert "not a tie" in index_mismatch("t", [0], [1], np.array([1.0, 4.0, 3.0]))
    assert index_mismatch("t", np.array([3, 1], dtype=np.int64), [1, 3]) == "t: idx [3, 1] vs oracle [1, 3]"
