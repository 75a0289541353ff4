"""Property-based pins of the oracle's element-level rounding (hypothesis):
for arbitrary bf16 magnitudes and fp32 block scales, on both grids, the
oracle's RTN / guided / SR choices equal exact rational search, and the
defining properties hold (guided picks a neighbour with the recorded bit,
SR picks one of the two neighbours).  No GPU is needed."""
from fractions import Fraction as F

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

E2M1 = [F(0), F(1, 2), F(1), F(3, 2), F(2), F(3), F(4), F(6)]
UNIFORM = [F(k) for k in range(8)]


def bf16(bits):
    return float((np.array([bits], np.uint32) << 16).view(np.float32)[0])


def f32(bits):
    return float(np.array([bits], np.uint32).view(np.float32)[0])


def nearest(grid, y):
    d = [abs(y - v) for v in grid]
    m = min(d)
    c = [j for j in range(8) if d[j] == m]
    return c[0] if len(c) == 1 else [j for j in c if j % 2 == 0][0]


def neighbours(grid, y):
    if y >= grid[7]:
        return 7, 7, True
    if y in grid:
        j = grid.index(y)
        return j, j, True
    lo = max(j for j in range(8) if grid[j] < y)
    return lo, lo + 1, False


# finite positive bf16 patterns and positive normal fp32 scales over a wide range
mag = st.integers(min_value=0, max_value=0x7F7F)
scale = st.integers(min_value=0x0C000000, max_value=0x72000000)


@pytest.mark.parametrize("fmt", [0, 2])
@settings(max_examples=400, deadline=None)
@given(h=mag, sb=scale, g=st.integers(0, 1), r=st.integers(0, (1 << 24) - 1))
def test_rounding_matches_rational_search(orc, fmt, h, sb, g, r):
    grid = E2M1 if fmt == 0 else UNIFORM
    ax, S = bf16(h), f32(sb)
    y = F(ax) / F(S)
    assert orc.rtn_code(fmt, ax, S) == nearest(grid, y)
    lo, hi, fixed = neighbours(grid, y)
    gd = orc.guided_code(fmt, ax, S, g)
    assert gd in (lo, hi)
    if not fixed:
        assert gd & 1 == g
    s = orc.sr_code(fmt, ax, S, r)
    assert s in (lo, hi)
    if not fixed:
        assert (s == hi) == (F(r) < (1 << 24) * (y - grid[lo]) / (grid[hi] - grid[lo]))


@settings(max_examples=300, deadline=None)
@given(h=mag, sb=scale)
def test_e2m1_rtn_equals_rounding_of_the_real_quotient_scaled_by_powers_of_two(orc, h, sb):
    """Scaling x and S by the same power of two does not change the code."""
    ax, S = bf16(h), f32(sb)
    for k in (-8, 3):
        ax2, S2 = ax * 2.0 ** k, S * 2.0 ** k
        if ax2 < 3.0e38 and S2 < 3.0e38 and np.float32(ax2) == ax2 and np.float32(S2) == S2 and S2 > 0:
            assert orc.rtn_code(0, ax2, S2) == orc.rtn_code(0, ax, S)
