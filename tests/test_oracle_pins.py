"""Pins for the CPU oracle: checks against things other than the oracle itself.

* hand-worked rows from the worked example of the RaZeR notes (golden file);
* library routines: torch float8_e4m3fn decode/encode (OCP E4M3, RNE),
  numpy float16 / torch bfloat16 rounding, numpy float32 division and a
  numpy float64 matmul;
* brute-force enumeration of every code assignment x every special value with
  exact rationals (fractions.Fraction) on tiny blocks;
* invariants of the method on synthetic config-like tensors.
"""
import itertools
import math
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

from bit_quantization_razer_b200 import workloads
from tests.golden_cases import case_tensor, load_cases

FMT = {"weight": 0, "act": 1, "nvfp4": 2}


def oracle_input(t: torch.Tensor):
    import oracle

    if t.dtype == torch.bfloat16:
        return oracle.Bf16Bits(workloads.to_numpy_bits(t))
    return t.numpy()


# ----------------------------------------------------------------------------
# hand-worked rows
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("case", load_cases(), ids=lambda c: c["name"])
def test_worked_rows(orc, case):
    fmt = FMT[case["fmt"]]
    x = case_tensor(case)
    xin = oracle_input(x)
    ts = orc.tensor_scale(xin, fmt)
    assert ts == case["ts"]
    codes, scales, ts2, _ = orc.quantize(xin, fmt)
    assert ts2 == case["ts"]
    np.testing.assert_array_equal(codes[0], case["codes"])
    np.testing.assert_array_equal(scales[0], case["scales"])
    deq = orc.dequant(codes, scales, ts, fmt, "f32")
    np.testing.assert_array_equal(deq[0], np.array(case["dequant"], np.float32))
    ones = np.ones((1, 32), np.float16)
    y = orc.gemm_ref(ones, codes, scales, ts, fmt)
    assert y[0, 0] == case["ones"]


# ----------------------------------------------------------------------------
# scale formats
# ----------------------------------------------------------------------------
def test_e4m3_decode_matches_torch(orc):
    codes = torch.arange(0, 127, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([orc.scale_value(1, int(c)) for c in range(127)])
    np.testing.assert_array_equal(got, ref)
    assert orc.scale_max(1) == 448.0 and orc.scale_max(2) == 448.0


def test_e3m3_decode(orc):
    vals = np.array([orc.scale_value(0, c) for c in range(64)])
    # anchors of an E3M3 / bias-3 format with subnormals
    assert vals[0x00] == 0.0 and vals[0x01] == 1 / 32 and vals[0x07] == 7 / 32
    assert vals[0x08] == 0.25 and vals[0x18] == 1.0 and vals[0x3F] == 30.0
    assert np.all(np.diff(vals) > 0)
    # the normal range (codes e >= 1) is the E4M3 grid on [0.25, 30]: E3M3
    # code (e, m) has the value of OCP E4M3 code (e + 4, m)
    e4 = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(8, 64):
        e, m = c >> 3, c & 7
        assert vals[c] == e4[((e + 4) << 3) | m]
    # subnormal spacing 1/32 continues into the first binade
    np.testing.assert_array_equal(np.diff(vals[:16]), np.full(15, 1 / 32))


def _adversarial_scales(hi: float, n_random: int, seed: int):
    rng = np.random.default_rng(seed)
    pts = set()
    e4 = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    grid = sorted(set(float(v) for v in e4 if v <= hi))
    for a, b in zip(grid[:-1], grid[1:]):
        mid = np.float32((a + b) / 2)
        for v in (mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9)), np.float32(a)):
            pts.add(float(v))
    pts.update(float(v) for v in rng.uniform(0, hi, n_random).astype(np.float32))
    pts.update([0.0, float(np.float32(1e-30)), hi])
    return sorted(pts)


def test_e4m3_encode_matches_torch(orc):
    # torch's float32 -> float8_e4m3fn conversion rounds to nearest even
    pts = _adversarial_scales(448.0, 4000, 0)
    t = torch.tensor(pts, dtype=torch.float32)
    ref = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.scale_encode(1, p) for p in pts], np.uint8)
    np.testing.assert_array_equal(got, ref)
    # above the largest code the nearest value is 448 itself
    for p in (448.5, 463.9, 464.0, 500.0, 1e30, float("inf")):
        assert orc.scale_encode(1, p) == 0x7E


def test_e3m3_encode(orc):
    pts = _adversarial_scales(30.0, 4000, 1)
    for p in pts:
        got = orc.scale_encode(0, p)
        if p >= 0.25:
            # normal range: same grid as E4M3 (torch RNE), code (e-4, m)
            c4 = int(torch.tensor([p], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])
            exp = (((c4 >> 3) - 4) << 3) | (c4 & 7)
            assert got == min(exp, 0x3F), p
        else:
            # subnormal range: round(32 p) with Python's half-to-even round()
            exp = round(Fraction(p) * 32)
            assert got == exp, p
    for p in (30.0, 30.999, 31.0, 32.0, 1e9):
        assert orc.scale_encode(0, p) == 0x3F


def test_e3m3_code_is_e4m3_code_of_sixteenth(orc):
    # the GPU quantizer encodes an E3M3 scale with the hardware E4M3 convert:
    # code = min(E4M3(s_f / 16), 63) -- the same grid scaled by 2^-4 in both
    # the normal and the subnormal range (torch's float32 -> E4M3 is RNE)
    pts = _adversarial_scales(30.0, 4000, 2) + [30.5, 31.0, 31.999]
    t = torch.tensor(pts, dtype=torch.float32) / 16
    c4 = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(int)
    for p, c in zip(pts, c4):
        assert orc.scale_encode(0, p) == min(c, 0x3F), p


# ----------------------------------------------------------------------------
# element grid
# ----------------------------------------------------------------------------
def test_fp4_grid(orc):
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        exp = mags[c & 7] * (-1 if c & 8 else 1)
        if c == 8:
            assert orc.fp4_value(c, None) == 0.0
            for v in (5.0, -5.0, 8.0, -8.0):
                assert orc.fp4_value(c, v) == v
        else:
            assert orc.fp4_value(c, None) == exp
            assert orc.fp4_value(c, 5.0) == exp
    assert [orc.special_value(0, m) for m in range(4)] == [5.0, -5.0, 8.0, -8.0]
    assert [orc.special_value(1, m) for m in range(2)] == [5.0, -5.0]
    assert orc.num_specials(2) == 0


# ----------------------------------------------------------------------------
# 16-bit conversions, tensor scale, division
# ----------------------------------------------------------------------------
def test_float_to_16bit_matches_libraries(orc):
    rng = np.random.default_rng(3)
    vals = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * np.float32(100),
        rng.standard_normal(1000).astype(np.float32) * np.float32(1e-6),
        np.array([0.0, -0.0, 65504.0, 1e-8, 6e-5, 2688.0, 0.1], np.float32),
    ])
    f16_ref = vals.astype(np.float16).view(np.uint16)
    bf_ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for v, a, b in zip(vals, f16_ref, bf_ref):
        assert orc.float_to_f16_bits(float(v)) == a
        assert orc.float_to_bf16_bits(float(v)) == b
    for h in range(0, 0x7C00, 7):
        assert orc.f16_to_double(h) == float(np.uint16(h).view(np.float16))


def test_tensor_scale(orc):
    w = workloads.weight(64, 256, seed=5)
    got = orc.tensor_scale(w.numpy(), 0)
    amax = np.abs(w.numpy().astype(np.float32)).max()
    assert got == np.float32(amax) / np.float32(180.0)
    a = workloads.outlier_activations(16, 256, seed=6)
    got = orc.tensor_scale(oracle_input(a), 1)
    amax = a.float().abs().max().item()
    assert got == np.float32(amax) / np.float32(2688.0)


def test_scaled_values_match_numpy_division(orc):
    rng = np.random.default_rng(4)
    for _ in range(300):
        x = (rng.standard_normal(16) * rng.uniform(0.001, 3)).astype(np.float32)
        ts = np.float32(rng.uniform(0.0001, 0.05))
        for fmt in (0, 1):
            codes, sb, xs, _ = orc.quantize_block(x, float(ts), fmt)
            sc = sb & (0x3F if fmt == 0 else 0x7F)
            s = np.float32(orc.scale_value(fmt, sc))
            # block scale code = nearest to amax / (6 ts) computed in fp32
            sf = np.float32(np.abs(x).max()) / np.float32(np.float32(6) * ts)
            assert sc == orc.scale_encode(fmt, float(sf))
            if sc:
                d = np.float32(s * ts)
                np.testing.assert_array_equal(xs, x / d)


# ----------------------------------------------------------------------------
# brute force over all code assignments with exact rationals
# ----------------------------------------------------------------------------
MAGS = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]


def _code_value(code, v):
    if code == 8:
        return v
    m = MAGS[code & 7]
    return -m if code & 8 else m


def brute_force_block(xs, specials):
    """Minimise the exact SSE over every (special value, code assignment);
    ties: lowest special index, then smaller magnitude per element (then the
    lower code, which makes 0 win over the plain -0 code).  Zero entries of
    xs are fixed to code 0 (the only zero-error code when v != 0)."""
    nz = [j for j in range(16) if xs[j] != 0]
    best = None
    metas = list(enumerate(specials)) if specials else [(0, None)]
    for meta, v in metas:
        vv = Fraction(v) if v is not None else Fraction(0)
        for assign in itertools.product(range(16), repeat=len(nz)):
            sse = Fraction(0)
            mags = []
            for j, c in zip(nz, assign):
                val = _code_value(c, vv)
                sse += (Fraction(float(xs[j])) - val) ** 2
                mags.append((abs(val), c))
            key = (sse, meta, mags)
            if best is None or key < best[0]:
                best = (key, meta, dict(zip(nz, assign)))
    _, meta, chosen = best
    codes = [chosen.get(j, 0) for j in range(16)]
    return meta, codes


ADV = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 4.5, 5.0, 5.5, 6.0, 7.0, 7.5, 8.0, 8.5, 9.0, 4.0, 3.0, 0.5]


def _tiny_blocks(seed, count, max_nz):
    rng = random.Random(seed)
    out = []
    for _ in range(count):
        n = rng.randint(1, max_nz)
        pos = rng.sample(range(16), n)
        xs = [0.0] * 16
        for p in pos:
            kind = rng.random()
            if kind < 0.5:
                a = rng.choice(ADV)
                a = float(np.float32(a))
                if rng.random() < 0.4:
                    a = float(np.nextafter(np.float32(a), np.float32(100 if rng.random() < 0.5 else 0)))
            else:
                a = float(np.float32(rng.uniform(0, 9)))
            xs[p] = a if rng.random() < 0.5 else -a
        out.append(xs)
    return out


@pytest.mark.parametrize("fmt,max_nz,count", [(0, 2, 150), (0, 3, 12), (1, 3, 40), (2, 3, 30)])
def test_bruteforce_tiny_blocks(orc, fmt, max_nz, count):
    specials = [orc.special_value(fmt, m) for m in range(orc.num_specials(fmt))]
    for xs_target in _tiny_blocks(100 + fmt * 10 + max_nz, count, max_nz):
        # realise X^scaled exactly with ts = 1/8 and a scale of 1/32 (weights:
        # subnormal E3M3, so |xs| may reach 9) or 1/64 (E4M3 formats), by
        # padding the block with an element that fixes the block amax
        if fmt == 0:
            d = Fraction(1, 32) / 8
        else:
            d = Fraction(1, 64) / 8
        x = [float(Fraction(t) * d) for t in xs_target]
        codes, sb, xs, _ = orc.quantize_block(np.array(x, np.float32), 0.125, fmt)
        s = orc.scale_value(fmt, sb & (0x3F if fmt == 0 else 0x7F))
        if s == 0:
            assert all(c == 0 for c in codes)
            continue
        meta_bf, codes_bf = brute_force_block(xs, specials)
        meta = (sb >> 6) if fmt == 0 else ((sb >> 7) if fmt == 1 else 0)
        assert meta == meta_bf, (xs, meta, meta_bf)
        assert list(codes) == codes_bf, (xs, list(codes), codes_bf)


# ----------------------------------------------------------------------------
# invariants on config-like tensors
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_invariants(orc, fmt):
    if fmt == 1:
        x = workloads.outlier_activations(64, 512, seed=11)
        xin = oracle_input(x)
        xf = x.float().numpy()
    else:
        x = workloads.weight(64, 512, seed=12)
        xin = x.numpy()
        xf = x.float().numpy()
    ts = orc.tensor_scale(xin, fmt)
    nv = orc.num_specials(fmt)
    specials = [orc.special_value(fmt, m) for m in range(nv)]
    max_xs = 0.0
    for r in range(0, 64, 3):
        for b in range(512 // 16):
            blk = xf[r, b * 16:(b + 1) * 16]
            codes, sb, xs, dl = orc.quantize_block(blk, ts, fmt)
            max_xs = max(max_xs, float(np.abs(xs).max()))
            sc = sb & (0x3F if fmt == 0 else 0x7F)
            meta = (sb >> 6) if fmt == 0 else ((sb >> 7) if fmt == 1 else 0)
            if fmt == 2:
                assert 8 not in codes  # 0b1000 never appears in plain NVFP4
                continue
            # the chosen value never raises the squared error over plain NVFP4
            assert dl[meta] <= 0.0
            assert dl[meta] == min(dl[:nv])
            a = np.abs(xs.astype(np.float64))
            in5 = (a > 4.5) & (a <= 5.5)
            in8 = a > 7
            if not (in5.any() or (fmt == 0 and in8.any())):
                assert meta == 0 and not np.any(dl[:nv])
                assert 8 not in codes
            # a code 0b1000 decodes to the chosen special value
            s = orc.scale_value(fmt, sc)
            for j in range(16):
                if codes[j] == 8:
                    assert orc.fp4_value(8, specials[meta]) * s == specials[meta] * s
                    assert abs(xs[j] - specials[meta]) <= 1.0
    # with a library-computed tensor scale X^scaled stays below 9 (+ rounding)
    assert max_xs <= 9.0 * (1 + 2 ** -20)


def test_gemm_ref_matches_numpy(orc):
    w = workloads.weight(48, 256, seed=21)
    codes, scales, ts, _ = orc.quantize(w.numpy(), 0)
    x = workloads.vectors(5, 256, seed=22)
    deq = orc.dequant(codes, scales, 1.0, 0, "f32").astype(np.float64)
    ref = (x.numpy().astype(np.float64) @ deq.T) * ts
    got = orc.gemm_ref(x.numpy(), codes, scales, ts, 0)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    sub = orc.gemm_ref(x.numpy(), codes, scales, ts, 0, rows=[4, 1])
    np.testing.assert_array_equal(sub, got[[4, 1]])


def test_dequant_output_types(orc):
    w = workloads.weight(8, 64, seed=23)
    codes, scales, ts, _ = orc.quantize(w.numpy(), 0)
    f32 = orc.dequant(codes, scales, ts, 0, "f32")
    f16 = orc.dequant(codes, scales, ts, 0, "f16")
    bf = orc.dequant(codes, scales, ts, 0, "bf16")
    np.testing.assert_array_equal(f16, f32.astype(np.float16).view(np.uint16))
    ref_bf = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bf, ref_bf)
    # q*s is exact; (q*s)*ts is one binary32 rounding
    qs = orc.dequant(codes, scales, 1.0, 0, "f32")
    np.testing.assert_array_equal(f32, qs * np.float32(ts))


def test_zero_and_degenerate(orc):
    z = np.zeros((2, 32), np.float16)
    codes, scales, ts, _ = orc.quantize(z, 0)
    assert ts == 0.0 and not codes.any() and not scales.any()
    # ts <= 0 given by the caller: all-zero output
    x = workloads.outlier_activations(2, 32, seed=1)
    codes, scales, _, _ = orc.quantize(oracle_input(x), 1, ts=0.0)
    assert not codes.any() and not scales.any()
    # a block of tiny values under a large tensor scale has scale code 0
    row = np.zeros((1, 32), np.float16)
    row[0, 0] = 1e-4
    row[0, 16] = 60000
    codes, scales, ts, _ = orc.quantize(row, 0)
    assert scales[0, 0] == 0 and codes[0, :8].sum() == 0
    with pytest.raises(ValueError):
        orc.quantize(np.zeros((1, 24), np.float16), 0)


@pytest.mark.parametrize("afmt,wfmt", [("act", "weight"), ("nvfp4", "nvfp4"), ("act", "act"), ("weight", "nvfp4")])
def test_w4a4_ref_matches_numpy(orc, afmt, wfmt):
    # with power-of-two tensor scales the f32 dequant (pinned above) is exact,
    # so a numpy float64 matmul of the two dequantized operands is the exact
    # product up to the summation order; random packed operands reach every
    # code, every meta value and the subnormal scale codes
    M, N, K = 9, 21, 96
    ca, sa = workloads.random_packed(M, K, afmt, seed=71)
    cw, sw = workloads.random_packed(N, K, wfmt, seed=72)
    ts_a, ts_w = 0.25, 2.0 ** -7
    A = orc.dequant(ca.numpy(), sa.numpy(), ts_a, FMT[afmt], "f32").astype(np.float64)
    W = orc.dequant(cw.numpy(), sw.numpy(), ts_w, FMT[wfmt], "f32").astype(np.float64)
    ref = A @ W.T
    got = orc.gemm_w4a4_ref(ca.numpy(), sa.numpy(), ts_a, FMT[afmt], cw.numpy(), sw.numpy(), ts_w, FMT[wfmt])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    sub = orc.gemm_w4a4_ref(ca.numpy(), sa.numpy(), ts_a, FMT[afmt], cw.numpy(), sw.numpy(), ts_w, FMT[wfmt], rows=[7, 0])
    np.testing.assert_array_equal(sub, got[[7, 0]])
    # one non-zero activation picks the weight column: a special code of A
    # (0b1000 -> its block's v) times W's dequantized column
    ca2 = np.zeros_like(ca.numpy())
    ca2[3, 5] = 0x80  # element 11 of row 3: code 0b1000
    sa2 = np.zeros_like(sa.numpy())
    sa2[3, 0] = (1 << 7 if afmt == "act" else 0) | 0x38  # meta 1 (-5 for activations), scale 1.0
    one = orc.gemm_w4a4_ref(ca2, sa2, 1.0, FMT[afmt], cw.numpy(), sw.numpy(), ts_w, FMT[wfmt])
    v = {"act": -5.0, "nvfp4": 0.0, "weight": None}[afmt]
    if v is not None:
        np.testing.assert_array_equal(one[3], v * W[:, 11])
        assert not one[[i for i in range(M) if i != 3]].any()


# ----------------------------------------------------------------------------
# accuracy ablations: FourOverSix and the quantization error
# ----------------------------------------------------------------------------
_E2M1_MAGS = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]


def _nearest_e2m1(xs: Fraction) -> tuple[int, Fraction]:
    # brute force over the 8 magnitudes, ties to the smaller magnitude (R7)
    a = abs(xs)
    best = min(range(8), key=lambda c: (abs(a - _E2M1_MAGS[c]), c))
    q = _E2M1_MAGS[best]
    code = best | (8 if xs < 0 and q != 0 else 0)
    return code, (-q if xs < 0 else q)


def _block_46_exact(x16: np.ndarray, ts: float, c: float):
    # library arithmetic for the float32 steps (numpy), torch for the E4M3
    # rounding, exact rationals for the rounding to the grid and the error
    amax = np.float32(np.max(np.abs(x16.astype(np.float32))))
    s_f = np.float32(amax / np.float32(np.float32(c) * np.float32(ts)))
    sc = int(torch.tensor([float(s_f)], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])
    sc = 0x7E if sc >= 0x7F else sc  # saturate
    s = float(torch.tensor([sc], dtype=torch.uint8).view(torch.float8_e4m3fn).float()[0])
    d = np.float32(np.float32(s) * np.float32(ts))
    xf = x16.astype(np.float32)
    if sc == 0 or d == 0:
        return [0] * 16, 0, sum(Fraction(float(v)) ** 2 for v in xf)
    codes, err = [], Fraction(0)
    for v in xf:
        xs = np.float32(v / d)
        code, q = _nearest_e2m1(Fraction(float(xs)))
        codes.append(code)
        err += (Fraction(float(v)) - q * Fraction(float(d))) ** 2
    return codes, sc, err


def test_four_over_six_bruteforce(orc):
    # blocks of varied spread; the exact choice (strictly smaller error takes
    # 4) against the oracle's double-precision one
    rng = np.random.default_rng(5)
    ts = 0.0037
    n_four = 0
    for trial in range(300):
        scale = 10.0 ** rng.uniform(-1, 1)
        x = (rng.standard_normal(16) * scale * (rng.random(16) ** rng.uniform(0, 3))).astype(np.float16)
        c6, s6, e6 = _block_46_exact(x, ts, 6.0)
        c4, s4, e4 = _block_46_exact(x, ts, 4.0)
        codes, scales, _, n4 = orc.quantize_46(x.reshape(1, 16), ts)
        got = [(codes[0, j // 2] >> (4 * (j & 1))) & 15 for j in range(16)]
        exp_codes, exp_sc = (c4, s4) if e4 < e6 else (c6, s6)
        assert got == exp_codes and int(scales[0, 0]) == exp_sc, trial
        assert n4 == (1 if e4 < e6 else 0)
        n_four += n4
    assert 0 < n_four < 300  # both choices occur


def test_quant_sse_and_ablation_invariants(orc):
    w = workloads.weight(64, 512, std=0.02, seed=31)
    # with a power-of-two tensor scale the f32 dequant (pinned above) is exact
    for fmt in (0, 2):
        codes, scales, _, _ = orc.quantize(w.numpy(), fmt, ts=2.0 ** -12)
        deq = orc.dequant(codes, scales, 2.0 ** -12, fmt, "f32").astype(np.float64)
        ref = float(np.sum((w.numpy().astype(np.float64) - deq) ** 2))
        assert math.isclose(orc.quant_sse(w.numpy(), codes, scales, 2.0 ** -12, fmt), ref, rel_tol=1e-12)
    # FourOverSix never does worse than plain NVFP4 (it includes its choice),
    # and the blocks that keep 6 are plain NVFP4 blocks
    cn, sn, ts, _ = orc.quantize(w.numpy(), 2)
    c46, s46, ts46, n4 = orc.quantize_46(w.numpy())
    assert ts46 == ts and n4 > 0
    assert orc.quant_sse(w.numpy(), c46, s46, ts, 2) < orc.quant_sse(w.numpy(), cn, sn, ts, 2)
    same = (s46 == sn)
    blocks6 = np.repeat(same, 8, axis=1)
    np.testing.assert_array_equal(c46[blocks6], cn[blocks6])


# ----------------------------------------------------------------------------
# format variants: block size and special-value set
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_generic_reduces_to_the_format(orc, fmt):
    # block 16 with the format's own special values is the format's quantizer
    w = workloads.weight(32, 256, std=0.02, seed=41)
    V = [orc.special_value(fmt, m) for m in range(orc.num_specials(fmt))]
    c, s, ts, _ = orc.quantize(w.numpy(), fmt)
    cg, sg, tg = orc.quantize_generic(w.numpy(), 16, fmt, V)
    assert tg == ts
    np.testing.assert_array_equal(cg, c)
    np.testing.assert_array_equal(sg, s)


def _brute_force_generic(xs, specials):
    # brute_force_block over any block length (zero entries fixed to code 0)
    nz = [j for j in range(len(xs)) if xs[j] != 0]
    best = None
    for meta, v in (list(enumerate(specials)) if specials else [(0, None)]):
        vv = Fraction(v) if v is not None else Fraction(0)
        for assign in itertools.product(range(16), repeat=len(nz)):
            sse = Fraction(0)
            mags = []
            for j, c in zip(nz, assign):
                val = _code_value(c, vv)
                sse += (Fraction(float(xs[j])) - val) ** 2
                mags.append((abs(val), c))
            key = (sse, meta, mags)
            if best is None or key < best[0]:
                best = (key, meta, dict(zip(nz, assign)))
    _, meta, chosen = best
    return meta, [chosen.get(j, 0) for j in range(len(xs))]


@pytest.mark.parametrize("bs,sfmt,V", [(32, 0, [2.5, -2.5, 7.0, -7.0]), (64, 1, [3.5, -3.5]), (32, 0, [5.5, -5.5, 9.5, -9.5])])
def test_generic_bruteforce(orc, bs, sfmt, V):
    # sparse blocks of length bs, X^scaled near the custom special values;
    # exact enumeration of (special value, codes) against the oracle
    rng = random.Random(bs + 7 * sfmt)
    ts = 0.125
    step = Fraction(1, 32) / 8 if sfmt == 0 else Fraction(1, 64) / 8
    checked = 0
    for _ in range(80):
        xs_t = [0.0] * bs
        for p in rng.sample(range(bs), rng.randint(1, 3)):
            a = float(np.float32(rng.choice([abs(V[0]) + d for d in (-0.6, -0.25, 0.0, 0.25, 0.6)] + [rng.uniform(0, 9.5)])))
            xs_t[p] = a if rng.random() < 0.5 else -a
        x = np.array([float(Fraction(t) * step) for t in xs_t], np.float32).reshape(1, bs)
        codes, scales, _ = orc.quantize_generic(x, bs, sfmt, V, ts=ts)
        sb = int(scales[0, 0])
        sc = sb & (0x3F if sfmt == 0 else 0x7F)
        got = [(int(codes[0, j // 2]) >> (4 * (j & 1))) & 15 for j in range(bs)]
        if sc == 0:
            assert not any(got)
            continue
        d = np.float32(np.float32(orc.scale_value(sfmt, sc)) * np.float32(ts))
        xs = [float(np.float32(np.float32(v) / d)) for v in x[0]]
        meta_bf, codes_bf = _brute_force_generic(xs, V)
        meta = sb >> (6 if sfmt == 0 else 7)
        assert meta == meta_bf and got == codes_bf, (xs, meta, meta_bf)
        checked += 1
    assert checked > 20


def test_quant_sse_generic_matches_python_decode(orc):
    # the error sum against a decode written here (value table + scale table)
    # and a numpy sum; block 64, custom pair on E4M3
    x = workloads.outlier_activations(8, 256, seed=43)
    V = [4.5, -4.5]
    codes, scales, ts = orc.quantize_generic(oracle_input(x), 64, 1, V)
    vals = np.zeros((8, 256))
    for r in range(8):
        for k in range(256):
            c = (int(codes[r, k // 2]) >> (4 * (k & 1))) & 15
            sb = int(scales[r, k // 64])
            q = V[sb >> 7] if c == 8 else _code_value(c, 0)
            vals[r, k] = float(q) * orc.scale_value(1, sb & 0x7F) * ts
    ref = float(np.sum((x.float().numpy().astype(np.float64) - vals) ** 2))
    got = orc.quant_sse_generic(oracle_input(x), 64, 1, V, codes, scales, ts)
    assert math.isclose(got, ref, rel_tol=1e-12)


def test_generic_f16_scale_bruteforce(orc):
    # the pages' kernel format (block 128, FP16 scale, meta in bits 15..14,
    # no tensor scale): the scale from numpy's float16 rounding, the choice
    # and codes by exact enumeration
    rng = random.Random(17)
    V = [5.0, -5.0, 8.0, -8.0]
    checked = 0
    for _ in range(30):
        s_true = float(np.float16(rng.uniform(0.01, 0.5)))
        xs_t = [0.0] * 128
        xs_t[rng.randrange(128)] = 6.0  # fixes the block amax
        for p in rng.sample(range(128), 2):
            a = rng.choice([4.6, 4.9, 5.2, 5.4, rng.uniform(0, 6)])
            xs_t[p] = a if rng.random() < 0.5 else -a
        x = np.array([np.float32(t * s_true) for t in xs_t], np.float32).reshape(1, 128)
        codes, scales, ts = orc.quantize_generic(x, 128, orc.SCALE_F16, V)
        assert ts == 1.0
        sw = int(scales[0, 0]) | (int(scales[0, 1]) << 8)
        h = int(np.float16(np.float32(np.max(np.abs(x))) / np.float32(6.0)).view(np.uint16))
        assert sw & 0x3FFF == min(h, 0x3FFF)
        d = np.float32(np.uint16(sw & 0x3FFF).view(np.float16))
        xs = [float(np.float32(v / d)) for v in x[0]]
        meta_bf, codes_bf = _brute_force_generic(xs, V)
        got = [(int(codes[0, j // 2]) >> (4 * (j & 1))) & 15 for j in range(128)]
        assert (sw >> 14) == meta_bf and got == codes_bf
        checked += 1
    assert checked == 30


# ----------------------------------------------------------------------------
# decoder and W4A16 reference of the format variants
# ----------------------------------------------------------------------------
_DEFAULT_V = {0: [5.0, -5.0, 8.0, -8.0], 1: [5.0, -5.0], 2: []}


def _random_scale_bytes(rng, shape, fmt):
    if fmt == 0:  # E3M3 magnitude (every 6-bit value valid) + 2 meta bits
        return rng.integers(0, 256, shape, dtype=np.uint8)
    mag = rng.integers(0, 0x7F, shape, dtype=np.uint8)  # E4M3 without the NaN code
    if fmt == 1:
        return mag | (rng.integers(0, 2, shape, dtype=np.uint8) << 7)
    return mag


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_dequant_generic_reduces_to_the_format(orc, fmt):
    # at block 16 with the format's own special values the variant decoder is
    # the pinned decoder; at blocks 32 / 128 it equals the pinned decoder on
    # scales repeated per 16 elements (the block index k / block)
    rng = np.random.default_rng(60 + fmt)
    R, K = 6, 256
    codes = rng.integers(0, 256, (R, K // 2), dtype=np.uint8)
    V = _DEFAULT_V[fmt]
    ts = 0.0123
    for bs in (16, 32, 128):
        sc = _random_scale_bytes(rng, (R, K // bs), fmt)
        sc16 = np.repeat(sc, bs // 16, axis=1)
        for odt in ("f32", "f16", "bf16"):
            np.testing.assert_array_equal(orc.dequant_generic(codes, sc, ts, bs, fmt, V, odt),
                                          orc.dequant(codes, sc16, ts, fmt, odt))


def test_dequant_generic_f16_scale_words(orc):
    # FP16 scale words: bits 13..0 read by numpy's float16 decode, the meta in
    # bits 15..14 selecting V like the E3M3 meta bits 7..6 (compared through an
    # E3M3 scale of exactly 1.0, code 0b011000), little-endian 16-bit words
    rng = np.random.default_rng(64)
    R, K, bs = 5, 384, 128
    V = [2.5, -7.0, 9.5, -3.5]
    codes = rng.integers(0, 256, (R, K // 2), dtype=np.uint8)
    mag = rng.integers(0, 0x4000, (R, K // bs), dtype=np.uint16)
    meta = rng.integers(0, 4, (R, K // bs), dtype=np.uint16)
    words = (mag | (meta << 14)).astype("<u2")
    got = orc.dequant_generic(codes, words.view(np.uint8), 1.0, bs, orc.SCALE_F16, V, "f32")
    unit = (24 | (meta.astype(np.uint8) << 6)).astype(np.uint8)
    q = orc.dequant_generic(codes, unit, 1.0, bs, 0, V, "f32").astype(np.float64)
    s = np.repeat(mag.view(np.float16).astype(np.float64), bs, axis=1)
    np.testing.assert_array_equal(got, (q * s).astype(np.float32))
    assert np.array_equal(q * s, (q * s).astype(np.float32).astype(np.float64))  # q*s exact in binary32


def test_gemv_generic_matches_numpy(orc):
    x = workloads.vectors(3, 256, seed=65)
    w = workloads.weight(40, 256, seed=66)
    for bs, sfmt, V in ((128, orc.SCALE_F16, [5.0, -5.0, 8.0, -8.0]), (32, 0, [5.0, -5.0, 7.0, -7.0]), (64, 1, [4.5, -4.5])):
        codes, scales, ts = orc.quantize_generic(w.numpy(), bs, sfmt, V)
        deq = orc.dequant_generic(codes, scales, 1.0, bs, sfmt, V, "f32").astype(np.float64)
        ref = (x.numpy().astype(np.float64) @ deq.T) * ts
        got = orc.gemv_generic(x.numpy(), codes, scales, ts, bs, sfmt, V)
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    # block 16 with the weight format's values is the pinned product reference
    codes, scales, ts, _ = orc.quantize(w.numpy(), 0)
    np.testing.assert_array_equal(orc.gemv_generic(x.numpy(), codes, scales, ts, 16, 0, _DEFAULT_V[0]),
                                  orc.gemm_ref(x.numpy(), codes, scales, ts, 0))


def test_dequant_generic_meta_past_the_set(orc):
    # a scale byte whose meta names no special value (never written by the
    # quantizer) decodes the 0b1000 code to 0 and leaves the other codes alone
    codes = np.full((1, 16), 0x18, np.uint8)  # nibbles 8 (low) and 1 (high): 0b1000, 0.5
    scales = np.array([[24 | (3 << 6), 24 | (1 << 6)]], np.uint8)  # E3M3 1.0, meta 3 / meta 1
    got = orc.dequant_generic(codes, scales, 1.0, 16, 0, [5.0, -5.0], "f32")
    np.testing.assert_array_equal(got[0, :16], np.tile([0.0, 0.5], 8).astype(np.float32))
    np.testing.assert_array_equal(got[0, 16:], np.tile([-5.0, 0.5], 8).astype(np.float32))


def _nearest_with_tie_rule(xs: Fraction, v):
    """Nearest point of Q_FP4 (and v when given) to xs; ties to the smaller
    magnitude.  Returns (value, code) with 0 encoded as 0b0000 and v as 0b1000."""
    cands = [(m, c) for c, m in enumerate(MAGS)] + [(-m, c | 8) for c, m in enumerate(MAGS) if m != 0]
    if v is not None:
        cands.append((Fraction(v), 8))
    best = min(cands, key=lambda pc: (abs(xs - pc[0]), abs(pc[0])))
    return best[0], (0 if best[0] == 0 else best[1])


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_full_blocks_exact_argmin(orc, fmt):
    # all 16 elements in play: given v each element's best point is
    # independent, so the exact SSE of every candidate is a sum of per-element
    # minima (rationals); the oracle's meta must be the argmin (ties: lowest
    # index) and its codes the nearest points under the tie rule
    rng = np.random.default_rng(70 + fmt)
    specials = [orc.special_value(fmt, m) for m in range(orc.num_specials(fmt))]
    mids = np.array(ADV, np.float32)
    checked, picks = 0, {}
    for i in range(300):
        x = rng.standard_normal(16).astype(np.float32)
        k = rng.integers(0, 8)  # some elements on grid midpoints (+-1 ulp) of xs
        x[:k] = rng.choice(mids, k) * rng.choice([-1.0, 1.0], k)
        x *= np.float32(rng.uniform(0.2, 1.5))
        if fmt == 0 and i % 2:
            # s_f just below a subnormal code midpoint, (m + 0.3..0.49) / 32 with
            # m = 1, 2: the scale rounds down to m / 32, so the block amax
            # lands at |xs| in (7, 9) and +-8 competes
            m = int(rng.integers(1, 3))
            ts = np.float32(np.abs(x).max() / (6 * (m + rng.uniform(0.3, 0.49)) / 32))
        else:
            ts = np.float32(rng.uniform(0.05, 0.5))
        codes, sb, xs, _ = orc.quantize_block(x, float(ts), fmt)
        if (sb & (0x3F if fmt == 0 else 0x7F)) == 0:
            assert all(c == 0 for c in codes)
            continue
        xsf = [Fraction(float(t)) for t in xs]
        sse = []
        for v in (specials or [None]):
            sse.append(sum((t - _nearest_with_tie_rule(t, v)[0]) ** 2 for t in xsf))
        meta = min(range(len(sse)), key=lambda m: (sse[m], m))
        got_meta = (sb >> 6) if fmt == 0 else ((sb >> 7) if fmt == 1 else 0)
        assert got_meta == meta, (i, sse)
        v = specials[meta] if specials else None
        assert list(codes) == [_nearest_with_tie_rule(t, v)[1] for t in xsf], i
        picks[meta] = picks.get(meta, 0) + 1
        checked += 1
    assert checked > 250
    if fmt == 0:
        assert picks.get(2, 0) + picks.get(3, 0) >= 10, picks  # +-8 really competes
