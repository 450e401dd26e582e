"""CPU proof of the byte-permute tables of the GEMV decoders.

prmt.b32 d, a, b, c (default mode) forms d byte by byte: nibble i of c
selects byte (c_i & 7) of the 8-byte pool {a bytes 0-3, b bytes 4-7}, and
bit 3 of the nibble replicates that byte's sign bit instead.  The decoders
build fp16 pairs [v(meta0), v(meta1)] of the special values and the scale
pairs with it; numpy's float16 gives the expected bit patterns.
"""
import numpy as np

V_W = [5.0, -5.0, 8.0, -8.0]  # meta 0..3 of the weight format


def prmt(a, b, c):
    pool = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    d = 0
    for i in range(4):
        sel = (c >> (4 * i)) & 0xF
        byte = pool[sel & 7]
        if sel & 8:
            byte = 0xFF if byte & 0x80 else 0x00
        d |= byte << (8 * i)
    return d


def f16(x):
    return int(np.float16(x).view(np.uint16))


def pair(lo, hi):
    return f16(lo) | (f16(hi) << 16)


def test_hot_path_special_value_pairs():
    # fp16 high bytes of +5, -5, +8, -8 (their low bytes are 0), indexed by meta
    k_vhigh = 0xC848C545
    for m0 in range(4):
        for m1 in range(4):
            sel = 0x0404 | (m0 << 4) | (m1 << 12)
            assert prmt(k_vhigh, 0, sel) == pair(V_W[m0], V_W[m1])


def test_variant_special_value_pairs():
    rng = np.random.default_rng(9)
    allowed = [h / 2 for h in range(5, 20) if h / 2 not in (3.0, 4.0, 6.0)]
    for _ in range(200):
        V = [float(v) * rng.choice([-1, 1]) for v in rng.choice(allowed, 4)]
        lo, hi = f16(V[0]) | (f16(V[1]) << 16), f16(V[2]) | (f16(V[3]) << 16)
        sel = lambda m: m * 0x22 + 0x10  # bytes 2m, 2m+1
        for m0 in range(4):
            assert prmt(lo, hi, sel(m0) * 0x101) == pair(V[m0], V[m0])
            for m1 in range(4):
                assert prmt(lo, hi, sel(m0) | (sel(m1) << 8)) == pair(V[m0], V[m1])


def test_scale_byte_spreading():
    for sb in (0x0000, 0x3F01, 0x12C7, 0xFFFF, 0x8040):
        x = prmt(sb, 0, 0x4140)  # 16-bit lanes: byte 0, byte 1
        assert x == (sb & 0xFF) | (((sb >> 8) & 0xFF) << 16)
        assert prmt(x, 0, 0x1010) == (x & 0xFFFF) * 0x10001   # low lane in both halves
        assert prmt(x, 0, 0x3232) == (x >> 16) * 0x10001      # high lane in both halves
