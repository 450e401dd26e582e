"""CPU proof of the +-5 candidate term the GPU quantizer relies on.

Adding v = 5 (for xs > 0; v = -5 mirrors it) to the E2M1 grid changes the
squared error of an element by

    d(xs) = (r5 - xs)^2 - (q - xs)^2,

where q is the nearest grid point and r5 the nearest point of the grid plus
5, both with ties to the smaller magnitude.  The kernel computes, in
binary32,

    t(xs) = sat(1 - |2|xs| - 10|)        (sat clamps to [0, 1])

with one saturating add, and uses d = -t.  This test checks d(xs) == -t(xs)
for EVERY binary32 in [4, 8) (d is computed exactly in float64 from its
definition) and that t vanishes on [2, 4) and [8, 16), where 5 is never the
nearest point.  Every t is a multiple of 2^-20 in [0, 1], so a block's 16
terms and their signed sums are exact binary32 sums in any order.

For blocks with a subnormal scale code (|xs| <= 9) the kernel also tries
v = 8, with the term min(28 - 4 xs, 0) from one FMA, and sums every term as
an integer in units of 2^-20; the last test checks that form on [2, 16).
"""
import numpy as np

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def nearest_ties_smaller(a, grid):
    """Nearest point of a sorted non-negative grid, ties to the smaller one."""
    idx = np.clip(np.searchsorted(grid, a), 1, len(grid) - 1)
    lo, hi = grid[idx - 1], grid[idx]
    r = np.where(a - lo <= hi - a, lo, hi)
    return np.where(a >= grid[-1], grid[-1], r)


def delta_exact(a32):
    a = a32.astype(np.float64)
    q = nearest_ties_smaller(a, GRID)
    r5 = nearest_ties_smaller(a, np.sort(np.append(GRID, 5.0)))
    return (r5 - a) ** 2 - (q - a) ** 2  # exact: a has 24 bits, the points few


def t_kernel(a32):
    u = np.float32(2) * a32                              # exact
    d = (u - np.float32(10)).astype(np.float32)          # one binary32 rounding
    s = (np.float32(1) - np.abs(d)).astype(np.float32)   # one binary32 rounding
    return np.clip(s, np.float32(0), np.float32(1))      # the saturation


def binade(lo_exp):
    start = np.float32(2.0 ** lo_exp).view(np.uint32)
    return (start + np.arange(1 << 23, dtype=np.uint32)).view(np.float32)


def test_candidate_term_exhaustive_4_to_8():
    a = binade(2)  # [4, 8)
    t = t_kernel(a)
    assert np.array_equal(delta_exact(a), -t.astype(np.float64))
    # multiples of 2^-20 in [0, 1]: 16 of them sum exactly in binary32
    scaled = t.astype(np.float64) * 2.0 ** 20
    assert np.array_equal(scaled, np.round(scaled)) and t.max() <= 1 and t.min() >= 0


def test_candidate_term_vanishes_outside():
    for e in (1, 3):  # [2, 4) and [8, 16)
        a = binade(e)
        assert not t_kernel(a).any()
        assert not delta_exact(a).any()


def test_candidate_term_values():
    a = np.array([4.5, 4.75, 5.0, 5.25, 5.5], np.float32)
    assert t_kernel(a).tolist() == [0.0, 0.5, 1.0, 0.5, 0.0]


def delta_exact_v(a32, v):
    a = a32.astype(np.float64)
    q = nearest_ties_smaller(a, GRID)
    r = nearest_ties_smaller(a, np.sort(np.append(GRID, v)))
    return (r - a) ** 2 - (q - a) ** 2


def t8_kernel(a32):
    return np.minimum((np.float64(-4) * a32.astype(np.float64) + 28.0).astype(np.float32), np.float32(0))


def t5_signed_kernel(a32):
    # the integer-sum form of the +5 term: min(|2 xs - 10| - 1, 0)
    e = (np.float32(2) * a32 - np.float32(10)).astype(np.float32)
    return np.minimum((np.abs(e) - np.float32(1)).astype(np.float32), np.float32(0))


def test_eight_term_exhaustive():
    for e in (1, 2, 3):  # [2, 16): every binary32
        a = binade(e)
        t8 = t8_kernel(a)
        assert np.array_equal(delta_exact_v(a, 8.0), t8.astype(np.float64))
        units = t8.astype(np.float64) * 2.0 ** 20
        assert np.array_equal(units, np.round(units))  # integers in units of 2^-20
        t5 = t5_signed_kernel(a)
        assert np.array_equal(delta_exact_v(a, 5.0), t5.astype(np.float64))
        units5 = t5.astype(np.float64) * 2.0 ** 20
        assert np.array_equal(units5, np.round(units5))
