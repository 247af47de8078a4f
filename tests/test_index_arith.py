"""The decode kernel's integer divisions by a run-time divisor are a multiply
and a shift: q = umulhi(i, floor((2^32 - 1) / d) + 1).  The kernel relies on
this being exact for every dividend it forms; checked here exhaustively
over those ranges (no GPU needed):
  - the x staging's item -> column, i / per_col with per_col = H / 8 for
    every H that is a multiple of 32 up to 32768, and every item index
    i < 8 * per_col (T <= 8 columns);
  - the slot table's entry -> column, i / k for k = 1..8 and i < 64.
"""
import numpy as np


def umulhi_div(i, d):
    m = np.uint64(0xFFFFFFFF // d + 1)
    return (i.astype(np.uint64) * m) >> np.uint64(32)


def test_item_column_division_is_exact():
    for H in range(32, 32768 + 1, 32):
        per_col = H // 8
        i = np.arange(8 * per_col, dtype=np.uint64)
        assert np.array_equal(umulhi_div(i, per_col), i // np.uint64(per_col)), H


def test_entry_column_division_is_exact():
    i = np.arange(64, dtype=np.uint64)
    for k in range(1, 9):
        assert np.array_equal(umulhi_div(i, k), i // np.uint64(k)), k
