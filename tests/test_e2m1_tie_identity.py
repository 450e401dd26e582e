"""CPU proof of the code-selection identity the GPU quantizer relies on.

The quantizer rounds X^scaled to the E2M1 grid with ties to the SMALLER
magnitude, but the hardware converter rounds ties to EVEN.  The kernel
converts both xs and pred(xs) = RN(xs * (1 - 2^-24)) (one ulp toward zero)
and keeps the odd code where they differ.  This test checks that rule
against the definition for every binary32 around every grid midpoint and a
large random sample (an exhaustive sweep of [0, 16] was run the same way).
Round-to-nearest-even is emulated exactly in float64 here.
"""
import numpy as np

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def rne_code(a):
    idx = np.clip(np.searchsorted(GRID, a), 1, 7)
    lo, hi = GRID[idx - 1], GRID[idx]
    code = np.where(a - lo < hi - a, idx - 1, idx)
    tie = (a - lo) == (hi - a)
    code = np.where(tie, np.where((idx - 1) % 2 == 0, idx - 1, idx), code)
    return np.where(a >= 6, 7, code)


def half_down_code(a):
    idx = np.clip(np.searchsorted(GRID, a), 1, 7)
    lo, hi = GRID[idx - 1], GRID[idx]
    code = np.where(a - lo <= hi - a, idx - 1, idx)
    return np.where(a >= 6, 7, code)


def check(a32):
    p32 = (a32 * np.float32(1 - 2.0 ** -24)).astype(np.float32)
    c1 = rne_code(a32.astype(np.float64))
    c2 = rne_code(p32.astype(np.float64))
    sel = np.where(c1 % 2 == 1, c1, c2)
    ref = half_down_code(a32.astype(np.float64))
    return int(np.count_nonzero(sel != ref))


def test_pred_is_one_ulp_toward_zero():
    rng = np.random.default_rng(0)
    a = rng.uniform(2.0 ** -20, 16, 200000).astype(np.float32)
    p = (a * np.float32(1 - 2.0 ** -24)).astype(np.float32)
    assert np.array_equal(p.view(np.uint32), a.view(np.uint32) - 1)


def test_identity_around_every_midpoint():
    bad = 0
    for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0):
        u = np.float32(m).view(np.uint32).astype(np.int64)
        a = np.arange(u - 65536, u + 65537, dtype=np.int64).astype(np.uint32).view(np.float32)
        bad += check(a)
    assert bad == 0


def test_identity_random_and_special():
    rng = np.random.default_rng(1)
    a = rng.uniform(0, 16, 2_000_000).astype(np.float32)
    special = np.array([0, 1e-40, 1e-30, 0.5, 1, 1.5, 2, 3, 4, 6, 8, 1e30], np.float32)
    assert check(np.concatenate([a, special])) == 0
