"""The comparison rules of tests/parity.py, checked on the CPU: each one
accepts what it should and rejects planted mistakes, so a GPU test that
passes through them says what it claims."""
from __future__ import annotations

import numpy as np
import pytest

from tests.parity import (check_against_fp64, check_exact_vs_dump, check_row_invariants,
                          check_scores_close)


def test_row_invariants():
    check_row_invariants(np.array([3, 5, 9]), 2, 10, 3)            # L = 8 >= k: k real entries
    check_row_invariants(np.array([10, 11, -1, -1]), 10, 12, 4)    # L = 2 < k: two real, then padding
    check_row_invariants(np.array([-1, -1]), 7, 7, 2)               # empty window: padding only
    bad = [
        (np.array([10, 10, -1, -1]), 10, 12, 4),   # duplicate
        (np.array([11, 10, -1, -1]), 10, 12, 4),   # not ascending
        (np.array([10, 12, -1, -1]), 10, 12, 4),   # outside [ks, ke)
        (np.array([10, 11, 0, -1]), 10, 12, 4),    # padding not -1
        (np.array([10, -1, -1, -1]), 10, 12, 4),   # fewer than min(k, L) real entries
    ]
    for idx, ks, ke, k in bad:
        with pytest.raises(AssertionError):
            check_row_invariants(idx, ks, ke, k)


def test_scores_close():
    I64 = np.array([1.0, -2.0, 0.0])
    E = np.array([10.0, 10.0, 1.0])
    check_scores_close(np.array([1.0009, -2.0009, 0.00009], dtype=np.float32), I64, E)
    with pytest.raises(AssertionError):
        check_scores_close(np.array([1.0011, -2.0, 0.0], dtype=np.float32), I64, E)


def _row():
    # scores of a window of 8 keys starting at key 100; the exact top-3 is
    # keys 103, 105, 101 (scores 9, 7, 5); key 106 ties closely with 101.
    I64 = np.array([1.0, 5.0, 2.0, 9.0, 0.0, 7.0, 4.9999, 3.0])
    E = np.full(8, 10.0)
    return I64, E


def test_against_fp64_accepts_the_exact_set_and_band_swaps():
    I64, E = _row()
    val = np.array([5.0, 9.0, 7.0], dtype=np.float32)
    assert check_against_fp64(np.array([101, 103, 105]), val, I64, E, 100, 3) == 1.0
    # 106 instead of 101: |4.9999 - 5| <= 1e-4 * (10 + 10)
    p = check_against_fp64(np.array([103, 105, 106]), np.array([9.0, 7.0, 4.9999], dtype=np.float32),
                           I64, E, 100, 3)
    assert p == pytest.approx(2 / 3)


def test_against_fp64_rejects_swaps_outside_the_band_and_wrong_scores():
    I64, E = _row()
    with pytest.raises(AssertionError):   # 107 (score 3) is far below the k-th score 5
        check_against_fp64(np.array([103, 105, 107]), None, I64, E, 100, 3)
    with pytest.raises(AssertionError):   # right set, one score off by 2e-3 * E
        check_against_fp64(np.array([101, 103, 105]), np.array([5.02, 9.0, 7.0], dtype=np.float32),
                           I64, E, 100, 3)
    with pytest.raises(AssertionError):   # padding value of a short window must be -inf
        check_against_fp64(np.array([100, 101, -1]), np.array([1.0, 5.0, 0.0], dtype=np.float32),
                           I64[:2], E[:2], 100, 3)


def test_exact_vs_dump_is_bit_exact():
    oidx = np.array([103, 105, 101, -1], dtype=np.int64)          # oracle: score order, then padding
    oval = np.array([9.0, 7.0, 0.0, -np.inf])
    gidx = np.array([101, 103, 105, -1], dtype=np.int32)          # GPU: ascending index order
    gval = np.array([0.0, 9.0, 7.0, -np.inf], dtype=np.float32)
    check_exact_vs_dump(gidx, gval, oidx, oval, 4)
    with pytest.raises(AssertionError):   # one index differs
        check_exact_vs_dump(np.array([101, 103, 104, -1], dtype=np.int32), gval, oidx, oval, 4)
    with pytest.raises(AssertionError):   # -0.0 where the dump has +0.0: bits differ
        check_exact_vs_dump(gidx, np.array([-0.0, 9.0, 7.0, -np.inf], dtype=np.float32), oidx, oval, 4)
    with pytest.raises(AssertionError):   # a value one ulp off
        check_exact_vs_dump(gidx, np.array([0.0, np.nextafter(np.float32(9), np.float32(10)), 7.0, -np.inf],
                                           dtype=np.float32), oidx, oval, 4)
