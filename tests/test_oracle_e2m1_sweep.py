"""Exhaustive pin of the oracle's E2M1 encoder: every binary32 value with
|v| <= 8, both signs.

The expected step function comes from the E2M1 grid alone (the 8 magnitudes
0, 0.5, 1, 1.5, 2, 3, 4, 6 that the pages give for the 1-2-1 element code):
round to nearest, a value exactly halfway between two neighbours takes the
neighbour with an even mantissa bit (the even code), and everything above 6
saturates to 6.  The sign bit is the input's, so -0 and the negative values
that round to zero give code 8.
"""
import numpy as np
import pytest

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def expected_runs(sign: int):
    """Run starts (bit patterns) and codes of round-to-nearest-even on the grid."""
    starts, codes = [0], [0]
    for c in range(1, 8):
        mid = np.float32((GRID[c - 1] + GRID[c]) / 2)        # exact in binary32
        # a tie goes to the even code: code c takes the midpoint itself when c is even
        first = mid if c % 2 == 0 else np.nextafter(mid, np.float32(np.inf))
        starts.append(int(np.array(first, np.float32).view(np.uint32)))
        codes.append(c)
    return np.array(starts, np.uint32), np.array(codes, np.uint8) | np.uint8(sign << 3)


@pytest.mark.parametrize("sign", [0, 1])
def test_oracle_e2m1_is_nearest_even_on_every_binary32_up_to_8(e2m1_oracle_runs, sign):
    starts, codes = e2m1_oracle_runs[sign]
    want_s, want_c = expected_runs(sign)
    assert starts.tolist() == want_s.tolist()
    assert codes.tolist() == want_c.tolist()
