"""GPU accuracy-ablation tools against the oracle: the FourOverSix quantizer
(bit-exact codes, scale bytes and tensor scale) and the quantization error
sum of packed tensors."""
import math

import numpy as np
import pytest
import torch

import bit_quantization_razer_b200 as R
from bit_quantization_razer_b200 import workloads
from tests.gpu_helpers import FMT_ID, cuda, oracle_in

pytestmark = [pytest.mark.gpu, cuda]
DEV = "cuda:0"


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_four_over_six_tiny_config(orc, dtype):
    # 256 x 512, N(0, 0.02^2) with 0.1% x10 outliers, plus rows of very
    # different spread so both choices and the zero / saturated scales occur
    w = workloads.weight(256, 512, std=0.02, seed=0, dtype=torch.float32)
    w[::7] *= 40.0
    w[3::11] *= 1e-4
    w[5] = 0.0
    w = w.to(dtype)
    oc, os_, ots, n4 = orc.quantize_46(oracle_in(w))
    c, s, t = R.razer_quantize_weights(w.to(DEV), "four_over_six")
    torch.cuda.synchronize()
    assert float(t.cpu()[0]) == ots
    np.testing.assert_array_equal(c.cpu().numpy(), oc)
    np.testing.assert_array_equal(s.cpu().numpy(), os_)
    assert 0 < n4 < 256 * 32


def test_four_over_six_full_size_sampled(orc):
    N, K = 4096, 4096
    w = workloads.weight(N, K, std=0.02, seed=77)
    ts = orc.tensor_scale(w.numpy(), FMT_ID["nvfp4"])
    c, s, t = R.razer_quantize_weights(w.to(DEV), "four_over_six")
    torch.cuda.synchronize()
    assert float(t.cpu()[0]) == ts
    rows = np.random.default_rng(3).choice(N, 40, replace=False)
    oc, os_, _, _ = orc.quantize_46(w[rows].numpy(), ts=ts)
    np.testing.assert_array_equal(c.cpu().numpy()[rows], oc)
    np.testing.assert_array_equal(s.cpu().numpy()[rows], os_)


@pytest.mark.parametrize("fmt", ["weight", "act", "nvfp4"])
def test_quant_error_matches_oracle(orc, fmt):
    # error sum of an oracle-quantized tensor (order of the partial sums
    # differs: relative 1e-12)
    x = workloads.outlier_activations(96, 1024, seed=78) if fmt == "act" else workloads.weight(96, 1024, seed=79)
    codes, scales, ts, _ = orc.quantize(oracle_in(x), FMT_ID[fmt])
    ref = orc.quant_sse(oracle_in(x), codes, scales, ts, FMT_ID[fmt])
    got = R.razer_quant_error(x.to(DEV), torch.from_numpy(codes).to(DEV), torch.from_numpy(scales).to(DEV),
                              torch.tensor([ts], dtype=torch.float32, device=DEV), fmt)
    assert math.isclose(float(got.cpu()[0]), ref, rel_tol=1e-12)


def test_ablation_weights_ordering():
    # the ablation on a decode-shape weight matrix: FourOverSix never loses to
    # plain NVFP4 (it contains NVFP4's choice); the three errors are finite
    w = workloads.weight(4096, 4096, std=0.02, seed=80).to(DEV)
    err = {}
    for fmt, dec in (("nvfp4", "nvfp4"), ("four_over_six", "nvfp4"), ("weight", "weight")):
        c, s, t = R.razer_quantize_weights(w, fmt)
        err[fmt] = float(R.razer_quant_error(w, c, s, t, dec).cpu()[0])
    assert err["four_over_six"] < err["nvfp4"]
    assert all(math.isfinite(v) and v > 0 for v in err.values())


VARIANTS = [(16, "weight", [5.0, -5.0, 8.0, -8.0]), (32, "weight", [2.5, -2.5, 7.0, -7.0]), (64, "act", [3.5, -3.5]),
            (128, "act", []), (128, "weight", [5.0, -5.0, 8.0, -8.0]), (32, "nvfp4", [4.5, -4.5]),
            (128, "f16_scale", [5.0, -5.0, 8.0, -8.0]), (64, "f16_scale", [])]


@pytest.mark.parametrize("block,sfmt,V", VARIANTS)
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_variant_matches_oracle(orc, block, sfmt, V, dtype):
    # rows of very different spread (subnormal scales, zero rows) so every
    # special value and the zero block occur
    w = workloads.weight(96, 1024, std=0.02, seed=81, dtype=torch.float32)
    w[::5] *= 30.0
    w[2::9] *= 1e-5
    w[7] = 0.0
    w = w.to(dtype)
    oc, os_, ots = orc.quantize_generic(oracle_in(w), block, FMT_ID[sfmt], V)
    c, s, t = R.razer_quantize_variant(w.to(DEV), block, sfmt, V)
    torch.cuda.synchronize()
    assert float(t.cpu()[0]) == ots
    np.testing.assert_array_equal(c.cpu().numpy(), oc)
    np.testing.assert_array_equal(s.cpu().numpy(), os_)
    ref = orc.quant_sse_generic(oracle_in(w), block, FMT_ID[sfmt], V, oc, os_, ots)
    got = float(R.razer_quant_error_variant(w.to(DEV), block, sfmt, V, c, s, t).cpu()[0])
    assert math.isclose(got, ref, rel_tol=1e-12)


def test_variant_block16_equals_fast_quantizer():
    # the variant path with the weight format's own set is the hot-path
    # quantizer, byte for byte, at a decode shape
    w = workloads.weight(4096, 4096, std=0.02, seed=82).to(DEV)
    c1, s1, t1 = R.razer_quantize_weights(w, "weight")
    c2, s2, t2 = R.razer_quantize_variant(w, 16, "weight", [5.0, -5.0, 8.0, -8.0])
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(s1, s2) and torch.equal(t1, t2)
