"""GPU GEMV (1 <= B <= 32) against the oracle's double-accumulated product."""
import numpy as np
import pytest
import torch

import bit_quantization_razer_b200 as R
from bit_quantization_razer_b200 import workloads
from tests.golden_cases import case_tensor, load_cases
from tests.gpu_helpers import FMT_ID, REL_TOL, assert_close_typed, cuda, oracle_in, rel_err

pytestmark = [pytest.mark.gpu, cuda]
DEV = "cuda:0"


def gemv(x, codes, scales, ts, fmt, out_dtype=torch.float32):
    y = R.razer_gemv(x.to(DEV), codes.to(DEV), scales.to(DEV), torch.tensor([ts], dtype=torch.float32, device=DEV),
                     fmt, out_dtype)
    torch.cuda.synchronize()
    return y


def test_worked_rows_ones(orc):
    # y = sum of the dequantized row with x = 1 (K = 128: four W1-style rows)
    for case in load_cases():
        if case["fmt"] == "act":
            continue
        row = case_tensor(case)
        w = row.repeat(1, 4)  # K = 128
        codes, scales, ts, _ = orc.quantize(oracle_in(w), FMT_ID[case["fmt"]])
        x = torch.ones(1, 128, dtype=torch.float16)
        y = gemv(x, torch.from_numpy(codes), torch.from_numpy(scales), ts, case["fmt"])
        assert float(y[0, 0]) == 4 * case["ones"]


@pytest.mark.parametrize("fmt", ["weight", "act", "nvfp4"])
@pytest.mark.parametrize("B", [1, 3, 8, 13, 16, 32])
@pytest.mark.parametrize("xdt", [torch.float16, torch.bfloat16])
def test_gemv_random_packed(orc, fmt, B, xdt):
    # random codes/scales cover every decode path, ragged N spans several row tiles
    N, K = 200, 1152
    codes, scales = workloads.random_packed(N, K, fmt, seed=40 + B)
    x = workloads.vectors(B, K, seed=41 + B, dtype=xdt)
    ts = 0.0371
    ref = orc.gemm_ref(oracle_in(x), codes.numpy(), scales.numpy(), ts, FMT_ID[fmt])
    y = gemv(x, codes, scales, ts, fmt)
    assert rel_err(y.cpu().numpy(), ref) <= REL_TOL


def test_gemv_tiny_config_quantized(orc):
    # config: W 256 x 512 fp16 quantized by the oracle, one fp16 vector, seed 0
    w = workloads.weight(256, 512, std=0.02, seed=0)
    codes, scales, ts, _ = orc.quantize(w.numpy(), 0)
    x = workloads.vectors(1, 512, seed=0)
    ref = orc.gemm_ref(x.numpy(), codes, scales, ts, 0)
    for odt in (torch.float32, torch.float16, torch.bfloat16):
        y = gemv(x, torch.from_numpy(codes), torch.from_numpy(scales), ts, "weight", odt)
        assert_close_typed(y, ref)


def test_gemv_one_hot_equals_dequant(orc):
    codes, scales = workloads.random_packed(64, 256, "weight", seed=50)
    ts = 0.25
    deq = orc.dequant(codes.numpy(), scales.numpy(), ts, 0, "f32")
    for k in (0, 1, 17, 130, 255):
        x = torch.zeros(1, 256, dtype=torch.float16)
        x[0, k] = 1.0
        y = gemv(x, codes, scales, ts, "weight").cpu().numpy()[0]
        np.testing.assert_array_equal(y, deq[:, k])


@pytest.mark.parametrize("N,K,B,fmt", [(4096, 4096, 1, "weight"), (4096, 4096, 4, "weight"), (14336, 4096, 16, "weight"),
                                       (4096, 14336, 1, "weight"), (4096, 14336, 16, "weight"), (8192, 8192, 1, "weight"),
                                       (8192, 8192, 8, "nvfp4"), (8192, 8192, 32, "weight"), (28672, 8192, 1, "weight"),
                                       (8192, 28672, 32, "weight"), (28672, 8192, 8, "nvfp4")])
def test_gemv_config_shapes(orc, N, K, B, fmt):
    # the decode (Llama-3-8B) and 70B projection shapes, 512 sampled output columns
    codes, scales = workloads.random_packed(N, K, fmt, seed=N + K + B, max_scale_code=40)
    x = workloads.vectors(B, K, seed=B)
    ts = 0.0045
    y = gemv(x, codes, scales, ts, fmt).cpu().numpy()
    cols = np.random.default_rng(1).choice(N, 512, replace=False)
    ref = orc.gemm_ref(x.numpy(), codes[cols].numpy(), scales[cols].numpy(), ts, FMT_ID[fmt])
    assert rel_err(y[:, cols], ref) <= REL_TOL


@pytest.mark.parametrize("fmt", ["weight", "act", "nvfp4"])
@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 9, 17, 32])
@pytest.mark.parametrize("xdt", [torch.float16, torch.bfloat16])
def test_gemv_tma_random_packed(orc, fmt, B, xdt):
    # K % 256 == 0 (bulk-tensor kernel): ragged N over three 128-row tiles,
    # 36 half-units shared unevenly by 36 CTAs
    N, K = 300, 1536
    codes, scales = workloads.random_packed(N, K, fmt, seed=140 + B)
    x = workloads.vectors(B, K, seed=141 + B, dtype=xdt)
    ts = 0.0371
    ref = orc.gemm_ref(oracle_in(x), codes.numpy(), scales.numpy(), ts, FMT_ID[fmt])
    y = gemv(x, codes, scales, ts, fmt)
    assert rel_err(y.cpu().numpy(), ref) <= REL_TOL


@pytest.mark.parametrize("N,K,B,fmt,xdt,odt", [(17, 16, 1, "weight", torch.float16, torch.float32),
                                               (200, 48, 3, "act", torch.bfloat16, torch.float16),
                                               (130, 144, 17, "nvfp4", torch.float16, torch.bfloat16),
                                               (64, 4112, 32, "weight", torch.bfloat16, torch.float32),
                                               (300, 400, 5, "weight", torch.float16, torch.float16)])
def test_gemv_generic_k(orc, N, K, B, fmt, xdt, odt):
    # K % 128 != 0 (the only K-shape error is K % 16 != 0): no 128-k chunking
    codes, scales = workloads.random_packed(N, K, fmt, seed=N + K + B, max_scale_code=40)
    x = workloads.vectors(B, K, seed=B + 7, dtype=xdt)
    ts = 0.0371
    ref = orc.gemm_ref(oracle_in(x), codes.numpy(), scales.numpy(), ts, FMT_ID[fmt])
    assert R.razer_workspace_size(R.RAZER_OP_GEMV, B, N, K) == 0
    y = gemv(x, codes, scales, ts, fmt, odt)
    assert_close_typed(y, ref)


@pytest.mark.parametrize("N,K,B", [(100, 256, 1), (128, 14336, 3), (129, 256, 2), (1, 4096, 1), (3000, 256, 7),
                                   (640, 2304, 32), (1280, 4096, 8)])
def test_gemv_stream_k_partitions(orc, N, K, B):
    # fewer half-units than SMs; one tile shared by 112 CTAs; a one-row tail
    # tile; N = 1; many tiles with one stage each; odd half-unit ranges
    codes, scales = workloads.random_packed(N, K, "weight", seed=N * 7 + K + B)
    x = workloads.vectors(B, K, seed=N + B)
    ts = 0.0123
    ref = orc.gemm_ref(x.numpy(), codes.numpy(), scales.numpy(), ts, 0)
    y1 = gemv(x, codes, scales, ts, "weight")
    y2 = gemv(x, codes, scales, ts, "weight")
    assert rel_err(y1.cpu().numpy(), ref) <= REL_TOL
    # the split-K partials are summed in a fixed order: repeat calls agree bit for bit
    assert torch.equal(y1, y2)


def test_gemv_workspace_garbage_and_reused(orc):
    # one workspace full of garbage (NaN bytes) through calls of different
    # shapes on both kernels (K % 256 == 0 and K % 256 == 128): its contents
    # on entry never leak into y
    shapes = [(4096, 4096, 4), (128, 14336, 2), (200, 1152, 3), (4096, 4096, 4), (300, 1536, 32)]
    need = max(R.razer_workspace_size(R.RAZER_OP_GEMV, B, N, K) for N, K, B in shapes)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=DEV)
    for i, (N, K, B) in enumerate(shapes):
        codes, scales = workloads.random_packed(N, K, "weight", seed=600 + i, max_scale_code=40)
        x = workloads.vectors(B, K, seed=610 + i)
        ts = torch.tensor([0.02], dtype=torch.float32, device=DEV)
        y = R.razer_gemv(x.to(DEV), codes.to(DEV), scales.to(DEV), ts, "weight", torch.float32, workspace=ws)
        torch.cuda.synchronize()
        assert R.razer_get_device_status() == 0
        cols = np.arange(0, N, max(1, N // 64))
        ref = orc.gemm_ref(x.numpy(), codes[cols].numpy(), scales[cols].numpy(), 0.02, 0)
        assert rel_err(y.cpu().numpy()[:, cols], ref) <= REL_TOL
        ws.fill_(0xFF)


def test_gemv_scales_only_4byte_aligned(orc):
    # a scale pointer that is 4- but not 16-byte aligned cannot back a tensor
    # map: the per-warp kernel serves the call (same results)
    N, K, B = 256, 1024, 2
    codes, scales = workloads.random_packed(N, K, "weight", seed=77)
    buf = torch.zeros(scales.numel() + 16, dtype=torch.uint8, device=DEV)
    sc = buf[4:4 + scales.numel()].view(N, K // 16)
    sc.copy_(scales.to(DEV))
    assert sc.data_ptr() % 16 == 4
    x = workloads.vectors(B, K, seed=78)
    y = R.razer_gemv(x.to(DEV), codes.to(DEV), sc, torch.tensor([0.5], device=DEV), "weight", torch.float32)
    torch.cuda.synchronize()
    ref = orc.gemm_ref(x.numpy(), codes.numpy(), scales.numpy(), 0.5, 0)
    assert rel_err(y.cpu().numpy(), ref) <= REL_TOL


def _batch_problem(N, K, B, fmt, seed, xdt=torch.float16, ts=0.0312):
    codes, scales = workloads.random_packed(N, K, fmt, seed=seed, max_scale_code=40)
    x = workloads.vectors(B, K, seed=seed + 1, dtype=xdt)
    return x, codes, scales, ts


@pytest.mark.parametrize("fmt", ["weight", "nvfp4"])
@pytest.mark.parametrize("xdt", [torch.float16, torch.bfloat16])
def test_gemv_batch_mixed(orc, fmt, xdt):
    # one call, every kind of problem: several of one n-tile class sharing a
    # launch (ragged N, tiles split between CTAs), B of every class, a K that
    # the bulk-tensor kernel does not take (K % 256 = 128: run on its own),
    # an empty K (y = 0) and an empty N
    specs = [(300, 512, 1), (1000, 256, 4), (130, 768, 8), (260, 1024, 16), (64, 1024, 32), (200, 384, 3), (70, 0, 2),
             (0, 256, 5), (520, 2048, 2)]
    probs = [_batch_problem(N, K, B, fmt, 100 + i, xdt, ts=0.02 + 0.01 * i) for i, (N, K, B) in enumerate(specs)]
    dev = [(x.to(DEV), c.to(DEV), s.to(DEV), torch.tensor([t], dtype=torch.float32, device=DEV)) for x, c, s, t in probs]
    ys = R.razer_gemv_batch(dev, fmt, torch.float32)
    torch.cuda.synchronize()
    for (x, c, s, t), y, (N, K, B) in zip(probs, ys, specs):
        assert y.shape == (B, N)
        if N == 0:
            continue
        if K == 0:
            assert not y.any()
            continue
        ref = orc.gemm_ref(oracle_in(x), c.numpy(), s.numpy(), t, FMT_ID[fmt])
        assert rel_err(y.cpu().numpy(), ref) <= REL_TOL, (N, K, B)


def test_gemv_batch_more_problems_than_a_launch(orc):
    # 11 problems of one class: two launches reuse the workspace; f16 output
    probs = [_batch_problem(128 + 64 * i, 256 * (1 + i % 3), 1 + i % 8, "weight", 200 + i) for i in range(11)]
    dev = [(x.to(DEV), c.to(DEV), s.to(DEV), torch.tensor([t], dtype=torch.float32, device=DEV)) for x, c, s, t in probs]
    ws = torch.full((R.razer_gemv_batch_workspace_size(dev),), 0xFF, dtype=torch.uint8, device=DEV)  # garbage
    ys = R.razer_gemv_batch(dev, "weight", torch.float16, workspace=ws)
    torch.cuda.synchronize()
    for (x, c, s, t), y in zip(probs, ys):
        assert_close_typed(y, orc.gemm_ref(x.numpy(), c.numpy(), s.numpy(), t, 0))


def test_gemv_batch_decode_projections_sampled(orc):
    # the Llama-3-8B decode GEMVs of one step (3 projections x B = 1, 4, 16)
    # in one call; 256 sampled output rows of each against the oracle
    specs = [(N, K, B) for N, K in [(4096, 4096), (14336, 4096), (4096, 14336)] for B in (1, 4, 16)]
    probs = [_batch_problem(N, K, B, "weight", 300 + i) for i, (N, K, B) in enumerate(specs)]
    dev = [(x.to(DEV), c.to(DEV), s.to(DEV), torch.tensor([t], dtype=torch.float32, device=DEV)) for x, c, s, t in probs]
    ys = R.razer_gemv_batch(dev, "weight", torch.float32)
    y2 = R.razer_gemv_batch(dev, "weight", torch.float32)
    torch.cuda.synchronize()
    for i, ((x, c, s, t), y, (N, K, B)) in enumerate(zip(probs, ys, specs)):
        assert torch.equal(y, y2[i])  # deterministic: same partition, same summation order
        rows = np.random.default_rng(i).choice(N, 256, replace=False)
        ref = orc.gemm_ref(x.numpy(), c.numpy()[rows], s.numpy()[rows], t, 0)
        assert rel_err(y.cpu().numpy()[:, rows], ref) <= REL_TOL


def test_gemv_bounded_wait_times_out_and_reports(orc):
    """One stage that the producer never fills (host-side fault injection):
    the consumers' bounded waits expire, the device status word reports
    RAZER_ERR_TIMEOUT, the kernel ends, and the next call is correct."""
    # 512 half-units over 148 CTAs: CTA 0 runs two stages, the second is skipped
    N, K, B = 256, 32768, 1
    codes, scales = workloads.random_packed(N, K, "weight", seed=95)
    x = workloads.vectors(B, K, seed=96)
    c, s, xd = codes.to(DEV), scales.to(DEV), x.to(DEV)
    ts = torch.ones(1, device=DEV)
    assert R.razer_get_device_status() == 0
    R.razer_debug_set_fault_injection(True)
    try:
        R.razer_gemv(xd, c, s, ts, "weight", torch.float32)
    finally:
        R.razer_debug_set_fault_injection(False)
    assert R.razer_get_device_status() == 7  # RAZER_ERR_TIMEOUT, read and cleared
    y = R.razer_gemv(xd, c, s, ts, "weight", torch.float32)
    torch.cuda.synchronize()
    assert R.razer_get_device_status() == 0
    ref = orc.gemm_ref(x.numpy(), codes.numpy(), scales.numpy(), 1.0, 0)
    assert rel_err(y.cpu().numpy(), ref) <= REL_TOL
