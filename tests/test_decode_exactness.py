"""CPU proof of the exactness facts the GPU decoders rely on.

* Placing a scale code's exponent and mantissa bits into the binary16 fields
  ((code & mask) << 7) gives exactly s * 2^-12 for E3M3 and s * 2^-8 for
  E4M3, subnormal codes included (the scale values come from the pinned
  oracle).
* q * s * 2^-bias is exact in fp16 for every code, scale code and special
  value the formats allow (the hot path's +-5 / +-8, and every variant value:
  a multiple of 0.5 in [2.5, 9.5]), so the decoded MMA operand is exact.
* In bf16 it is exact for the hot-path values and for every variant value
  except +-9.5 (19 times a scale significand of 15 needs 9 bits; 8.5 gives at
  most 17 * 15 = 255), which is why the variant GEMV refuses +-9.5 with bf16
  activations.
* Every q (no scale) is exact in fp16 and bf16 (the FP16-scale-word GEMV
  multiplies the exact q and scales afterwards).
"""
import numpy as np
import torch

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
VARIANT_V = [h / 2 for h in range(5, 20) if h / 2 not in (3.0, 4.0, 6.0)]


def _is_fp16(x):
    return np.float64(np.float16(x)) == x


def _is_bf16(x):
    return float(torch.tensor(x, dtype=torch.float64).to(torch.bfloat16).to(torch.float64)) == x


def test_scale_bits_place_the_scale(orc):
    for fmt, mask, bias in ((0, 0x3F, 12), (1, 0x7F, 8)):
        for c in range(mask + 1):
            if fmt == 1 and c == 0x7F:
                continue  # E4M3 NaN code, never written
            bits = np.uint16((c & mask) << 7)
            assert float(bits.view(np.float16)) == orc.scale_value(fmt, c) * 2.0 ** -bias, (fmt, c)


def test_products_exact_in_fp16(orc):
    for fmt, ncodes, bias in ((0, 64, 12), (1, 127, 8)):
        scales = [orc.scale_value(fmt, c) * 2.0 ** -bias for c in range(ncodes)]
        values = E2M1 + [5.0, 8.0] + VARIANT_V
        for s in scales:
            for q in values:
                assert _is_fp16(q * s) and _is_fp16(-q * s), (fmt, s, q)


def test_products_in_bf16(orc):
    rounds = {9.5}
    for fmt, ncodes, bias in ((0, 64, 12), (1, 127, 8)):
        scales = [orc.scale_value(fmt, c) * 2.0 ** -bias for c in range(ncodes)]
        for q in E2M1 + [5.0, 8.0] + VARIANT_V:
            exact = all(_is_bf16(q * s) for s in scales)
            assert exact == (q not in rounds), (fmt, q)


def test_q_alone_exact_in_both_types():
    for q in E2M1 + [5.0, 8.0] + VARIANT_V:
        assert _is_fp16(q) and _is_bf16(q)
