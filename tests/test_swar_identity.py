"""CPU proof of the packed-nibble (SWAR) steps of the GPU decoders and the
quantizer.

* Redundant-zero indicator (GEMV / GEMM decode): for a word w of 8 codes,
  t = (w & 0x77777777) + 0x77777777 sets bit 3 of a nibble exactly when its
  low three bits are non-zero (no carry leaves a nibble: 7 + 7 < 16), so
  w & ~t & 0x88888888 marks the nibbles equal to 0b1000; the high half of
  its product with 2^30 is that mask shifted right by 2, i.e. the E2M1 code
  of 1.0 (0b0010) in exactly those nibbles.
* Region test (quantizer): after v = codes ^ 0x33333333,
  ~(((v & 0x77777777) + 0x77777777) | v) & 0x88888888 marks the nibbles whose
  code was 0b0011.
Each nibble is independent, so every nibble value in every position plus a
random sample of words covers the identities.
"""
import numpy as np

M7 = np.uint64(0x77777777)
M8 = np.uint64(0x88888888)
MASK32 = np.uint64(0xFFFFFFFF)


def nibbles(w):
    return [(w >> np.uint64(4 * i)) & np.uint64(15) for i in range(8)]


def words():
    rng = np.random.default_rng(5)
    w = [rng.integers(0, 2 ** 32, 200000, dtype=np.uint64)]
    for pos in range(8):  # every nibble value at every position, over random backgrounds
        base = rng.integers(0, 2 ** 32, 16, dtype=np.uint64) & ~np.uint64(15 << (4 * pos))
        w.append(base | (np.arange(16, dtype=np.uint64) << np.uint64(4 * pos)))
    return np.concatenate(w)


def test_indicator_marks_code_1000():
    w = words()
    t = ((w & M7) + M7) & MASK32
    is8 = w & ~t & M8 & MASK32
    ind = (is8 * np.uint64(2 ** 30)) >> np.uint64(32)  # umulhi(is8, 2^30)
    assert np.array_equal(ind, is8 >> np.uint64(2))
    for i, nib in enumerate(nibbles(w)):
        got = (ind >> np.uint64(4 * i)) & np.uint64(15)
        assert np.array_equal(got, np.where(nib == 8, 2, 0).astype(np.uint64))


def test_region_marks_code_0011():
    w = words()
    v = w ^ np.uint64(0x33333333)
    mark = ~(((v & M7) + M7) | v) & M8 & MASK32
    for i, nib in enumerate(nibbles(w)):
        got = (mark >> np.uint64(4 * i)) & np.uint64(15)
        assert np.array_equal(got, np.where(nib == 3, 8, 0).astype(np.uint64))
