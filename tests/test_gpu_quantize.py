"""GPU quantizer and decoder against the CPU oracle: codes, scale bytes, meta
bits and the tensor scale must match bit for bit; dequantized values too."""
import numpy as np
import pytest
import torch

import bit_quantization_razer_b200 as R
from bit_quantization_razer_b200 import workloads
from tests.golden_cases import case_tensor, load_cases
from tests.gpu_helpers import FMT_ID, cuda, oracle_in

pytestmark = [pytest.mark.gpu, cuda]
DEV = "cuda:0"


@pytest.fixture(params=["two_pass", "single_pass"])
def qpath(request):
    """Runs a dynamic-scale test once per quantizer path (both must give the
    oracle's bits)."""
    prev = R.razer_set_quantize_path(request.param)
    try:
        yield request.param
    finally:
        R.razer_set_quantize_path(prev)


@pytest.fixture
def single_pass():
    prev = R.razer_set_quantize_path("single_pass")
    try:
        yield
    finally:
        R.razer_set_quantize_path(prev)


def quantize_gpu(x: torch.Tensor, fmt: str, ts_in=None):
    x = x.to(DEV)
    if fmt == "act":
        c, s, t, h = R.razer_quantize_acts(x, ts_in, fmt)
    elif fmt == "act_nvfp4":
        c, s, t, h = R.razer_quantize_acts(x, ts_in, "nvfp4", hist=False)
    else:
        c, s, t = R.razer_quantize_weights(x, fmt)
        h = None
    torch.cuda.synchronize()
    return c.cpu().numpy(), s.cpu().numpy(), float(t.cpu()[0]), (None if h is None else h.cpu().numpy())


@pytest.mark.parametrize("case", load_cases(), ids=lambda c: c["name"])
def test_worked_rows_gpu(orc, case):
    x = case_tensor(case)
    fmt = case["fmt"]
    c, s, t, _ = quantize_gpu(x, fmt if fmt != "nvfp4" else "nvfp4")
    assert t == case["ts"]
    np.testing.assert_array_equal(c[0], case["codes"])
    np.testing.assert_array_equal(s[0], case["scales"])
    ts = torch.tensor([t], device=DEV)
    deq = R.razer_dequant(torch.from_numpy(c).to(DEV), torch.from_numpy(s).to(DEV), ts, fmt, torch.float32)
    np.testing.assert_array_equal(deq.cpu().numpy()[0], np.array(case["dequant"], np.float32))


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("fmt", ["weight", "nvfp4"])
def test_quantize_weights_tiny_config(orc, dtype, fmt, qpath):
    # 256 x 512, N(0, 0.02^2), 0.1% x10 outliers, seed 0
    w = workloads.weight(256, 512, std=0.02, seed=0, dtype=dtype)
    oc, os_, ots, _ = orc.quantize(oracle_in(w), FMT_ID[fmt])
    c, s, t, _ = quantize_gpu(w, fmt)
    assert t == ots
    np.testing.assert_array_equal(c, oc)
    np.testing.assert_array_equal(s, os_)


@pytest.mark.parametrize("N,K", [(4096, 4096), (14336, 4096), (4096, 14336)])
def test_quantize_weights_llama8b_sampled(orc, N, K):
    w = workloads.weight(N, K, std=0.02, seed=200 + N // 1024 + K // 1024)
    ots = orc.tensor_scale(w.numpy(), 0)
    c, s, t, _ = quantize_gpu(w, "weight")
    assert t == ots
    rows = np.random.default_rng(N + K).choice(N, 48, replace=False)
    oc, os_, _, _ = orc.quantize(w[rows].numpy(), 0, ts=ots)
    np.testing.assert_array_equal(c[rows], oc)
    np.testing.assert_array_equal(s[rows], os_)
    # the special values are in use, and +-8 only under subnormal scale codes
    meta = s >> 6
    assert (meta == 1).any() and (meta == 0).any()
    assert not ((meta >= 2) & ((s & 0x3F) >= 8)).any()


def test_quantize_weights_subnormal_scales(orc):
    # rows whose blocks mostly have subnormal E3M3 scale codes (tiny blocks
    # next to one huge element), so that +8 / -8 compete with +5 / -5
    g = torch.Generator().manual_seed(7)
    w = (torch.rand(64, 512, generator=g) * 2 - 1) * 0.3
    w[:, ::64] = 180.0
    w[::2, 1::64] = -180.0
    w = w.to(torch.float16)
    oc, os_, ots, _ = orc.quantize(w.numpy(), 0)
    c, s, t, _ = quantize_gpu(w, "weight")
    assert t == ots
    np.testing.assert_array_equal(s, os_)
    np.testing.assert_array_equal(c, oc)
    assert ((s >> 6) >= 2).any()


def _subnormal_rows():
    g = torch.Generator().manual_seed(11)
    w = (torch.rand(48, 256, generator=g) * 2 - 1) * 0.3
    w[:, ::64] = 180.0
    w[::2, 1::64] = -180.0
    return w


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("fmt", ["weight", "nvfp4"])
def test_quantize_weights_batch_vs_oracle(orc, dtype, fmt):
    # ragged row counts, an empty matrix inside the batch, a matrix whose
    # blocks use subnormal scale codes (+-8 in play) and one larger than the
    # next, so every stage mixes quantization and amax work of unequal size
    Ws = [workloads.weight(256, 512, std=0.02, seed=21, dtype=dtype),
          workloads.weight(100, 256, std=0.5, seed=22, dtype=dtype),
          torch.empty(0, 64, dtype=dtype),
          _subnormal_rows().to(dtype),
          workloads.weight(7, 2048, std=3.0, seed=23, dtype=dtype)]
    codes, scales, ts = R.razer_quantize_weights_batch([w.to(DEV) for w in Ws], fmt)
    torch.cuda.synchronize()
    ts = ts.cpu().numpy()
    for i, w in enumerate(Ws):
        oc, os_, ots, _ = orc.quantize(oracle_in(w), FMT_ID[fmt])
        assert ts[i] == np.float32(ots), i
        np.testing.assert_array_equal(codes[i].cpu().numpy(), oc.reshape(codes[i].shape))
        np.testing.assert_array_equal(scales[i].cpu().numpy(), os_.reshape(scales[i].shape))


def test_quantize_weights_batch_llama8b_equals_single_calls(orc):
    # the decode-step projections in one batch: every byte equals the
    # separate calls' output, ts equals the oracle's, sampled rows the oracle's
    shapes = [(4096, 4096), (14336, 4096), (4096, 14336)]
    Ws = [workloads.weight(N, K, std=0.02, seed=300 + i).to(DEV) for i, (N, K) in enumerate(shapes)]
    codes, scales, ts = R.razer_quantize_weights_batch(Ws, "weight")
    for i, w in enumerate(Ws):
        c1, s1, t1 = R.razer_quantize_weights(w, "weight")
        torch.cuda.synchronize()
        assert torch.equal(codes[i], c1) and torch.equal(scales[i], s1)
        assert float(ts[i]) == float(t1[0])
        wc = w.cpu()
        ots = orc.tensor_scale(wc.numpy(), 0)
        assert float(ts[i]) == ots
        rows = np.random.default_rng(i).choice(w.shape[0], 16, replace=False)
        oc, os_, _, _ = orc.quantize(wc[rows].numpy(), 0, ts=ots)
        np.testing.assert_array_equal(codes[i].cpu().numpy()[rows], oc)
        np.testing.assert_array_equal(scales[i].cpu().numpy()[rows], os_)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_quantize_acts_dynamic(orc, dtype, qpath):
    x = workloads.outlier_activations(256, 4096, seed=300, dtype=dtype)
    oc, os_, ots, oh = orc.quantize(oracle_in(x), 1)
    c, s, t, h = quantize_gpu(x, "act")
    assert t == ots
    np.testing.assert_array_equal(c, oc)
    np.testing.assert_array_equal(s, os_)
    np.testing.assert_array_equal(h, oh[[0, 1, 4, 5]].astype(np.int64))


def test_quantize_acts_single_pass_matches_given_scale(single_pass):
    # the single-pass kernel (dynamic scale; every SM's slice in shared memory)
    # against the streaming quantizer given the same scale: the full tensor,
    # bit for bit, with the histogram
    x = workloads.outlier_activations(2048, 4096, seed=305)
    c1, s1, t1, h1 = quantize_gpu(x, "act")
    ts_in = torch.tensor([t1], dtype=torch.float32, device=DEV)
    c2, s2, t2, h2 = quantize_gpu(x, "act", ts_in=ts_in)
    assert t2 == t1
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(h1, h2)


@pytest.mark.parametrize("M,K", [(1, 148 * 16), (3, 149 * 16), (37, 4096), (1, 147 * 16)])
def test_quantize_acts_small_slices(orc, M, K, qpath):
    # one block per SM, one SM with one more block, ragged slices, fewer
    # blocks than SMs (the single-pass path hands that to the two-pass one)
    x = workloads.outlier_activations(M, K, seed=M + K)
    oc, os_, ots, oh = orc.quantize(oracle_in(x), 1)
    c, s, t, h = quantize_gpu(x, "act")
    assert t == ots
    np.testing.assert_array_equal(c, oc)
    np.testing.assert_array_equal(s, os_)
    np.testing.assert_array_equal(h, oh[[0, 1, 4, 5]].astype(np.int64))


def test_quantize_single_pass_barrier_times_out_and_reports(orc, single_pass):
    """One CTA that never reaches the grid barrier (host-side fault
    injection): the others' bounded waits expire, the device status word
    reports RAZER_ERR_TIMEOUT, and the next call is correct."""
    x = workloads.outlier_activations(256, 4096, seed=306)
    assert R.razer_get_device_status() == 0
    R.razer_debug_set_fault_injection(True)
    try:
        quantize_gpu(x, "act")
    finally:
        R.razer_debug_set_fault_injection(False)
    assert R.razer_get_device_status() == 7  # RAZER_ERR_TIMEOUT, read and cleared
    oc, os_, ots, _ = orc.quantize(oracle_in(x), 1)
    c, s, t, _ = quantize_gpu(x, "act")
    assert R.razer_get_device_status() == 0
    assert t == ots
    np.testing.assert_array_equal(c, oc)
    np.testing.assert_array_equal(s, os_)


def test_quantize_acts_full_config_sampled(orc, qpath):
    # 2048 tokens x 4096, rows N(0,1), 8 channels x50, bf16
    x = workloads.outlier_activations(2048, 4096, seed=301)
    xin = oracle_in(x)
    ots = orc.tensor_scale(xin, 1)
    c, s, t, h = quantize_gpu(x, "act")
    assert t == ots
    rows = np.random.default_rng(5).choice(2048, 32, replace=False)
    oc, os_, _, _ = orc.quantize(oracle_in(x[rows]), 1, ts=ots)
    np.testing.assert_array_equal(c[rows], oc)
    np.testing.assert_array_equal(s[rows], os_)
    assert h[0] + h[1] == 2048 * 4096 // 16
    assert h[2] <= h[0] and h[3] <= h[1]


def test_quantize_acts_static_scale(orc):
    x = workloads.outlier_activations(64, 1024, seed=302)
    for ts_val in (0.05, 1e-4, 3.0, 0.0):
        oc, os_, _, oh = orc.quantize(oracle_in(x), 1, ts=ts_val)
        ts_in = torch.tensor([ts_val], dtype=torch.float32, device=DEV)
        c, s, t, h = quantize_gpu(x, "act", ts_in=ts_in)
        assert t == np.float32(ts_val)
        np.testing.assert_array_equal(c, oc)
        np.testing.assert_array_equal(s, os_)
        np.testing.assert_array_equal(h, oh[[0, 1, 4, 5]].astype(np.int64))


def test_quantize_acts_static_scale_huge_bf16(orc):
    # a caller-given ts far below the data: every block scale saturates and
    # X^scaled of the blocks scaled by 2^100 overflows binary32 (inf, rounded
    # to +-6 like any value above the grid); ts = 2^-60 is inside the
    # launch-wide fast range, 2^-80 outside it with divisors still inside the
    # corrected-reciprocal range
    x = workloads.outlier_activations(64, 1024, seed=304).float()
    x[::3, 16:48] *= 2.0 ** 100
    x[1::5, 512:528] *= -(2.0 ** 120)
    x = x.to(torch.bfloat16)
    for ts_val in (2.0 ** -60, 2.0 ** -80):
        oc, os_, _, oh = orc.quantize(oracle_in(x), 1, ts=ts_val)
        ts_in = torch.tensor([ts_val], dtype=torch.float32, device=DEV)
        c, s, t, h = quantize_gpu(x, "act", ts_in=ts_in)
        np.testing.assert_array_equal(c, oc)
        np.testing.assert_array_equal(s, os_)
        np.testing.assert_array_equal(h, oh[[0, 1, 4, 5]].astype(np.int64))


def test_quantize_acts_nvfp4(orc):
    x = workloads.outlier_activations(64, 1024, seed=303)
    oc, os_, ots, _ = orc.quantize(oracle_in(x), 2)
    c, s, t, h = R.razer_quantize_acts(x.to(DEV), None, "nvfp4", hist=False)
    assert float(t.cpu()[0]) == ots
    np.testing.assert_array_equal(c.cpu().numpy(), oc)
    np.testing.assert_array_equal(s.cpu().numpy(), os_)


def test_quantize_edge_cases(orc):
    # all zeros -> ts = 0, zero codes and scales
    z = torch.zeros(32, 64, dtype=torch.float16)
    c, s, t, _ = quantize_gpu(z, "weight")
    assert t == 0.0 and not c.any() and not s.any()
    # a single row, a single block
    w = workloads.weight(1, 16, seed=9)
    oc, os_, ots, _ = orc.quantize(w.numpy(), 0)
    c, s, t, _ = quantize_gpu(w, "weight")
    assert t == ots
    np.testing.assert_array_equal(c, oc)
    np.testing.assert_array_equal(s, os_)
    # empty tensor: nothing written but ts
    e = torch.empty(0, 64, dtype=torch.float16, device=DEV)
    c, s, t = R.razer_quantize_weights(e)
    assert float(t.cpu()[0]) == 0.0
    # ragged row count with a large dynamic range (denormal fp16 inputs)
    w = workloads.weight(37, 96, seed=10)
    w[3, :16] = torch.tensor(6e-8, dtype=torch.float16)
    w[5, 16:32] = 0
    oc, os_, ots, _ = orc.quantize(w.numpy(), 0)
    c, s, t, _ = quantize_gpu(w, "weight")
    np.testing.assert_array_equal(c, oc)
    np.testing.assert_array_equal(s, os_)


def test_bad_arguments_raise():
    x = torch.zeros(4, 24, dtype=torch.float16, device=DEV)
    with pytest.raises(R.RazerError) as e:
        R.razer_quantize_weights(x)
    assert "SHAPE" in str(e.value)
    x = torch.zeros(4, 32, dtype=torch.float32, device=DEV)
    with pytest.raises(R.RazerError):
        R.razer_quantize_weights(x)


@pytest.mark.parametrize("fmt", ["weight", "act", "nvfp4"])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_dequant_bit_exact(orc, fmt, out_dtype):
    codes, scales = workloads.random_packed(96, 256, fmt, seed=11, max_scale_code=None)
    ts = np.float32(0.0123)
    if out_dtype != torch.float32:
        ts = np.float32(0.5)  # keep every value inside the fp16 range
    ref = orc.dequant(codes.numpy(), scales.numpy(), float(ts), FMT_ID[fmt],
                      {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[out_dtype])
    out = R.razer_dequant(codes.to(DEV), scales.to(DEV), torch.tensor([ts], device=DEV), fmt, out_dtype)
    got = out.cpu()
    if out_dtype == torch.float32:
        np.testing.assert_array_equal(got.numpy(), ref)
    else:
        np.testing.assert_array_equal(workloads.to_numpy_bits(got), ref)
