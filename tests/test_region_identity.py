"""CPU proof of the special-value region test the GPU quantizer relies on.

For the +-5 candidates the quantizer needs, per element, whether
|xs| lies in (4.5, 5.5] (the elements whose nearest point changes when 5 is
added to the grid).  The kernel computes y = RN(|xs| / 2 - (1 + 2^-23)) with
one fused multiply-add and converts y to E2M1 with the hardware converter
(round to nearest, ties to even): the element is in the region exactly when
that code is 0b0011 (1.5), i.e. when 1.25 < y < 1.75.

This test checks the equivalence for EVERY binary32 |xs| in [4, 8), and on
the neighbouring binades [2, 4) and [8, 16) that the code is never 0b0011
there.  Below 2 and above 16, y lies below 0 or above 7, far from
(1.25, 1.75).  The fused multiply-add is emulated exactly: |xs| / 2 and
1 + 2^-23 are binary32 values whose difference float64 holds exactly, and the
single rounding to binary32 is numpy's RNE conversion.
"""
import numpy as np

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def e2m1_rne_code(a):
    """Magnitude code of the hardware E2M1 convert: nearest grid point, ties to
    the even code, saturating at 6."""
    idx = np.clip(np.searchsorted(GRID, a), 1, 7)
    lo, hi = GRID[idx - 1], GRID[idx]
    code = np.where(a - lo < hi - a, idx - 1, idx)
    tie = (a - lo) == (hi - a)
    code = np.where(tie, np.where((idx - 1) % 2 == 0, idx - 1, idx), code)
    return np.where(a >= 6, 7, code)


def region_by_kernel(a32):
    y = (a32.astype(np.float64) * 0.5 - (1.0 + 2.0 ** -23)).astype(np.float32)  # one rounding
    return e2m1_rne_code(y.astype(np.float64)) == 3


def binade(lo_exp):
    """Every binary32 in [2^lo_exp, 2^(lo_exp + 1))."""
    start = np.float32(2.0 ** lo_exp).view(np.uint32)
    return (start + np.arange(1 << 23, dtype=np.uint32)).view(np.float32)


def test_region_exhaustive_4_to_8():
    for e in (2,):  # [4, 8): 2^23 values
        a = binade(e)
        want = (a > np.float32(4.5)) & (a <= np.float32(5.5))
        got = region_by_kernel(a)
        assert np.array_equal(got, want)
        assert want.sum() == 1 << 21  # (4.5, 5.5] holds 2^21 binary32 values (spacing 2^-21)


def test_region_never_outside():
    for e in (1, 3):  # [2, 4) and [8, 16)
        assert not region_by_kernel(binade(e)).any()


def test_region_boundaries():
    a = np.array([4.5, np.nextafter(np.float32(4.5), np.float32(8)), 5.0, 5.5, np.nextafter(np.float32(5.5), np.float32(8))],
                 np.float32)
    assert region_by_kernel(a).tolist() == [False, True, True, True, False]
