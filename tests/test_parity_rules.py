"""CPU checks of the parity rules the GPU tests apply (tests/parity.py)."""
import numpy as np

from tests import parity as P


def test_index_row_validation():
    nb = np.array([5, 10, 2])
    good = np.array([[0, 1, 2, 4], [1, 3, 5, 9], [0, 1, -1, -1]], dtype=np.int32)
    assert P.check_index_rows(good, nb, 4) == []
    bad = good.copy()
    bad[0] = [0, 2, 1, 4]          # not ascending
    bad[1] = [1, 3, 5, 10]         # out of range
    bad[2] = [0, -1, -1, -1]       # wrong count
    assert P.check_index_rows(bad, nb, 4) == [0, 1, 2]


def test_selection_rule():
    s = np.array([0.9, 0.5, 0.50005, 0.1, 0.3], dtype=np.float32)
    ora = np.array([[0, 2]], dtype=np.int32)
    kth = np.array([[0.50005, 0.5]], dtype=np.float32)
    # exact
    r = P.compare_selection(ora.copy(), ora, kth, lambda i: s)
    assert r["exact"] == [0] and not r["bad"]
    # swapped within the tie band
    r = P.compare_selection(np.array([[0, 1]], dtype=np.int32), ora, kth, lambda i: s)
    assert r["tie"] == [0] and not r["bad"]
    # swapped outside the band
    r = P.compare_selection(np.array([[0, 4]], dtype=np.int32), ora, kth, lambda i: s)
    assert r["bad"]
    # a wide gap allows no difference at all
    kth2 = np.array([[0.9, 0.3]], dtype=np.float32)
    r = P.compare_selection(np.array([[1, 2]], dtype=np.int32), np.array([[0, 2]], dtype=np.int32), kth2,
                            lambda i: s)
    assert r["bad"]


def test_output_tolerance():
    a = np.array([0x3F80, 0x4000], dtype=np.uint16)       # 1.0, 2.0
    assert P.output_errors(a, a) == (0.0, 0.0)
    b = np.array([0x3F81, 0x4000], dtype=np.uint16)       # 1.0078125
    mx, mean = P.output_errors(b, a)
    assert abs(mx - 2 ** -7) < 1e-12 and abs(mean - 2 ** -8) < 1e-12
    nan = np.array([0x7FC0, 0x4000], dtype=np.uint16)
    assert P.output_errors(nan, a)[0] == float("inf")
