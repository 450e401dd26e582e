"""tcgen05 GEMM against the oracle's double-accumulated product."""
import numpy as np
import pytest
import torch

import bit_quantization_razer_b200 as R
from bit_quantization_razer_b200 import workloads
from tests.gpu_helpers import FMT_ID, REL_TOL, assert_close_typed, cuda, oracle_in, rel_err

pytestmark = [pytest.mark.gpu, cuda]
DEV = "cuda:0"


def gemm(X, codes, scales, ts, fmt, out_dtype=torch.float32):
    Y = R.razer_gemm(X.to(DEV), codes.to(DEV), scales.to(DEV), torch.tensor([ts], dtype=torch.float32, device=DEV),
                     fmt, out_dtype)
    torch.cuda.synchronize()
    assert R.razer_get_device_status() == 0
    return Y


def test_gemm_small_single_tile(orc):
    M, N, K = 128, 256, 128
    codes, scales = workloads.random_packed(N, K, "weight", seed=70, max_scale_code=40)
    X = workloads.vectors(M, K, seed=71, dtype=torch.bfloat16)
    ref = orc.gemm_ref(oracle_in(X), codes.numpy(), scales.numpy(), 0.25, 0)
    Y = gemm(X, codes, scales, 0.25, "weight")
    assert rel_err(Y.cpu().numpy(), ref) <= REL_TOL


@pytest.mark.parametrize("M", [1, 8, 33, 129])
def test_gemm_fewer_rows_than_a_tile(orc, M):
    # M below the 128-row TMA box of the activations (the rows past M read
    # as zeros) and 8192 columns of K split over several CTAs per tile
    N, K = 512, 8192
    codes, scales = workloads.random_packed(N, K, "weight", seed=84 + M, max_scale_code=40)
    X = workloads.vectors(M, K, seed=85, dtype=torch.bfloat16)
    ref = orc.gemm_ref(oracle_in(X), codes.numpy(), scales.numpy(), 0.03125, 0)
    Y = gemm(X, codes, scales, 0.03125, "weight")
    assert rel_err(Y.cpu().numpy(), ref) <= REL_TOL


@pytest.mark.parametrize("M", [200, 300])
@pytest.mark.parametrize("fmt", ["weight", "act", "nvfp4"])
@pytest.mark.parametrize("xdt", [torch.bfloat16, torch.float16])
def test_gemm_ragged_multi_tile(orc, fmt, xdt, M):
    # M tail (200 rows: the fused in-shared-memory decode; 300 rows: the
    # decode-once path), N not a multiple of 32, 3 k-steps (one pass over the
    # stages)
    N, K = 272, 192
    codes, scales = workloads.random_packed(N, K, fmt, seed=72, max_scale_code=None)
    X = workloads.vectors(M, K, seed=73, dtype=xdt)
    ts = 0.0371
    ref = orc.gemm_ref(oracle_in(X), codes.numpy(), scales.numpy(), ts, FMT_ID[fmt])
    Y = gemm(X, codes, scales, ts, fmt)
    assert rel_err(Y.cpu().numpy(), ref) <= REL_TOL


@pytest.mark.parametrize("M,rows", [(4096, 32), (200, 200)])
def test_gemm_oracle_quantized_weights_full_size(orc, M, rows):
    # a realistic 4096 x 4096 weight matrix (N(0, 0.02^2), 0.1% x10 outliers)
    # quantized by the oracle, at the prefill M (persistent decode-once path,
    # sampled rows) and at M = 200 (fused decode, every row)
    w = workloads.weight(4096, 4096, std=0.02, seed=123)
    codes, scales, ts, _ = orc.quantize(w.numpy(), 0)
    X = workloads.vectors(M, 4096, seed=124, dtype=torch.bfloat16)
    Y = gemm(X, torch.from_numpy(codes), torch.from_numpy(scales), ts, "weight", torch.float32).cpu().numpy()
    sel = np.sort(np.random.default_rng(125).choice(M, rows, replace=False))
    ref = orc.gemm_ref(oracle_in(X[sel]), codes, scales, ts, 0)
    assert rel_err(Y[sel], ref) <= REL_TOL


@pytest.mark.parametrize("M", [240, 512])
def test_gemm_oracle_quantized_weights(orc, M):
    # realistic weights quantized by the oracle; 8 k-steps wrap the 3-stage
    # ring (M = 240: fused decode, M = 512: decode-once)
    w = workloads.weight(512, 512, std=0.02, seed=74)
    codes, scales, ts, _ = orc.quantize(w.numpy(), 0)
    X = workloads.vectors(M, 512, seed=75, dtype=torch.bfloat16)
    ref = orc.gemm_ref(oracle_in(X), codes, scales, ts, 0)
    for odt in (torch.float32, torch.bfloat16, torch.float16):
        Y = gemm(X, torch.from_numpy(codes), torch.from_numpy(scales), ts, "weight", odt)
        assert_close_typed(Y, ref)


def test_gemm_one_hot_rows_equal_dequant(orc):
    codes, scales = workloads.random_packed(256, 128, "weight", seed=76)
    deq = orc.dequant(codes.numpy(), scales.numpy(), 0.5, 0, "f32")
    X = torch.zeros(256, 128, dtype=torch.bfloat16)
    for m in range(256):
        X[m, m % 128] = 1.0
    Y = gemm(X, codes, scales, 0.5, "weight").cpu().numpy()
    for m in (0, 5, 127, 128, 200, 255):
        np.testing.assert_array_equal(Y[m], deq[:, m % 128])


@pytest.mark.parametrize("M,N,K,rows", [(4096, 4096, 4096, 96), (4096, 14336, 4096, 24), (2048, 4096, 14336, 24)])
def test_gemm_prefill_shapes_sampled(orc, M, N, K, rows):
    codes, scales = workloads.random_packed(N, K, "weight", seed=M + N + K, max_scale_code=40)
    X = workloads.vectors(M, K, seed=77, dtype=torch.bfloat16)
    ts = 0.0045
    Y = gemm(X, codes, scales, ts, "weight").cpu().numpy()
    sel = np.sort(np.random.default_rng(2).choice(M, rows, replace=False))
    ref = orc.gemm_ref(oracle_in(X[sel]), codes.numpy(), scales.numpy(), ts, 0)
    assert rel_err(Y[sel], ref) <= REL_TOL


def test_gemm_k_zero_and_errors():
    codes = torch.zeros(32, 0, dtype=torch.uint8, device=DEV)
    scales = torch.zeros(32, 0, dtype=torch.uint8, device=DEV)
    X = torch.zeros(8, 0, dtype=torch.bfloat16, device=DEV)
    Y = R.razer_gemm(X, codes, scales, torch.ones(1, device=DEV), "weight", torch.float32)
    torch.cuda.synchronize()
    assert not Y.any()
    with pytest.raises(R.RazerError):  # K % 16
        R.razer_gemm(torch.zeros(8, 24, dtype=torch.bfloat16, device=DEV), torch.zeros(48, 12, dtype=torch.uint8, device=DEV),
                     torch.zeros(48, 2, dtype=torch.uint8, device=DEV), torch.ones(1, device=DEV))


@pytest.mark.parametrize("M,N,K,fmt,xdt,odt", [(1, 17, 16, "weight", torch.bfloat16, torch.float32),
                                               (100, 40, 80, "act", torch.float16, torch.float16),
                                               (33, 100, 208, "nvfp4", torch.bfloat16, torch.bfloat16),
                                               (300, 24, 16400, "weight", torch.bfloat16, torch.float32),
                                               (1100, 18, 144, "weight", torch.float16, torch.float16),
                                               (130, 300, 1040, "weight", torch.bfloat16, torch.bfloat16)])
def test_gemm_generic_shapes(orc, M, N, K, fmt, xdt, odt):
    # K % 64 != 0 and N % 16 != 0 (rows not 16-byte aligned, a ragged last
    # k-step, a K spanning two accumulation chains, M above the decode-once
    # threshold) against the oracle
    codes, scales = workloads.random_packed(N, K, fmt, seed=M + N + K, max_scale_code=40)
    X = workloads.vectors(M, K, seed=M + 1, dtype=xdt)
    ts = 0.0213
    Y = R.razer_gemm(X.to(DEV), codes.to(DEV), scales.to(DEV), torch.tensor([ts], device=DEV), fmt, odt)
    torch.cuda.synchronize()
    rows = np.arange(M) if M <= 256 else np.random.default_rng(M).choice(M, 64, replace=False)
    ref = orc.gemm_ref(oracle_in(X[rows]), codes.numpy(), scales.numpy(), ts, FMT_ID[fmt])
    assert_close_typed(Y[rows], ref)


@pytest.mark.parametrize("M,N,K", [(50, 24, 80), (7, 100, 16)])
def test_gemm_w4a4_generic_shapes(orc, M, N, K):
    xa = workloads.vectors(M, K, seed=M, dtype=torch.bfloat16)
    ca, sa, ta, _ = R.razer_quantize_acts(xa.to(DEV), None, "act", hist=False)
    cw, sw = workloads.random_packed(N, K, "weight", seed=N + K, max_scale_code=40)
    tw = torch.tensor([0.031], device=DEV)
    Y = R.razer_gemm_w4a4(ca, sa, ta, cw.to(DEV), sw.to(DEV), tw, "act", "weight", torch.float32)
    torch.cuda.synchronize()
    ref = orc.gemm_w4a4_ref(ca.cpu().numpy(), sa.cpu().numpy(), float(ta.cpu()[0]), 1, cw.numpy(), sw.numpy(), 0.031, 0)
    assert rel_err(Y.cpu().numpy(), ref) <= REL_TOL


def test_gemm_bounded_wait_times_out_and_reports():
    """A decoder warp that never arrives (host-side fault injection) makes the
    MMA thread's bounded wait expire: the kernel stops, frees its tensor
    memory, and the device status word reports RAZER_ERR_TIMEOUT; the context
    stays usable."""
    codes, scales = workloads.random_packed(256, 64, "weight", seed=90)
    X = workloads.vectors(128, 64, seed=91, dtype=torch.bfloat16).to(DEV)  # M < 256: the fused kernel
    c, s = codes.to(DEV), scales.to(DEV)
    ts = torch.ones(1, device=DEV)
    assert R.razer_get_device_status() == 0
    R.razer_debug_set_fault_injection(True)
    try:
        R.razer_gemm(X, c, s, ts, "weight", torch.float32)
    finally:
        R.razer_debug_set_fault_injection(False)
    assert R.razer_get_device_status() == 7  # RAZER_ERR_TIMEOUT, read and cleared
    assert R.razer_get_device_status() == 0
    # the next call works normally
    Y = R.razer_gemm(X, c, s, ts, "weight", torch.float32)
    torch.cuda.synchronize()
    import oracle
    ref = oracle.gemm_ref(oracle_in(X.cpu()), codes.numpy(), scales.numpy(), 1.0, 0)
    assert rel_err(Y.cpu().numpy(), ref) <= REL_TOL


def test_gemm_persistent_bounded_wait_times_out_and_reports():
    """The decode-once path's persistent kernel: one CTA never fills its first
    stage (host-side fault injection), the MMA issuer's bounded wait expires,
    every role stops, the tensor memory is freed and the status word reports
    RAZER_ERR_TIMEOUT; the next call is correct."""
    M, N, K = 1024, 512, 256
    codes, scales = workloads.random_packed(N, K, "weight", seed=92)
    X = workloads.vectors(M, K, seed=93, dtype=torch.bfloat16).to(DEV)
    c, s = codes.to(DEV), scales.to(DEV)
    ts = torch.ones(1, device=DEV)
    assert R.razer_get_device_status() == 0
    R.razer_debug_set_fault_injection(True)
    try:
        R.razer_gemm(X, c, s, ts, "weight", torch.float32)
    finally:
        R.razer_debug_set_fault_injection(False)
    assert R.razer_get_device_status() == 7
    assert R.razer_get_device_status() == 0
    Y = R.razer_gemm(X, c, s, ts, "weight", torch.float32)
    torch.cuda.synchronize()
    import oracle
    rows = np.arange(0, M, 37)
    ref = oracle.gemm_ref(oracle_in(X.cpu()[rows]), codes.numpy(), scales.numpy(), 1.0, 0)
    assert rel_err(Y.cpu().numpy()[rows], ref) <= REL_TOL


@pytest.mark.parametrize("M,N,K", [(1024, 256, 64), (1280, 640, 192), (4096, 4096, 512), (1100, 300, 128), (1024, 258, 4096)])
def test_gemm_persistent_units(M, N, K):
    """Unit walk of the persistent kernel: fewer units than SMs, several
    units per CTA with ragged last tiles (M, N not multiples of 256), and
    rows of N % 4 != 0 elements (scalar stores); every row is checked."""
    codes, scales = workloads.random_packed(N, K, "weight", seed=M + N + K, max_scale_code=40)
    X = workloads.vectors(M, K, seed=94, dtype=torch.bfloat16)
    ts = torch.tensor([0.02], device=DEV)
    Y = R.razer_gemm(X.to(DEV), codes.to(DEV), scales.to(DEV), ts, "weight", torch.float32)
    torch.cuda.synchronize()
    import oracle
    ref = oracle.gemm_ref(oracle_in(X), codes.numpy(), scales.numpy(), 0.02, 0)
    assert rel_err(Y.cpu().numpy(), ref) <= REL_TOL
    # the bf16 output is the fp32 result rounded once
    Yb = R.razer_gemm(X.to(DEV), codes.to(DEV), scales.to(DEV), ts, "weight", torch.bfloat16)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Yb.cpu().float().numpy(), torch.from_numpy(Y.cpu().numpy()).to(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("M,N,K,fmt", [(512, 28672, 8192, "weight"), (2048, 8192, 28672, "weight"), (8192, 8192, 8192, "nvfp4"),
                                       (1024, 4096, 4096, "act")])
def test_gemm_70b_sweep_sampled(orc, M, N, K, fmt):
    # the 70B projection shapes of the sweep (M = 512 runs the fused decode,
    # M >= 1024 the decode-once path); 32 sampled output rows against the oracle
    codes, scales = workloads.random_packed(N, K, fmt, seed=M + N + K, max_scale_code=40)
    X = workloads.vectors(M, K, seed=79, dtype=torch.bfloat16)
    ts = 0.0031
    Y = gemm(X, codes, scales, ts, fmt).cpu().numpy()
    sel = np.sort(np.random.default_rng(3).choice(M, 32, replace=False))
    ref = orc.gemm_ref(oracle_in(X[sel]), codes.numpy(), scales.numpy(), ts, FMT_ID[fmt])
    assert rel_err(Y[sel], ref) <= REL_TOL


@pytest.mark.parametrize("xdt", [torch.float16, torch.bfloat16])
def test_gemm_decoded_path_f16_and_garbage_workspace(orc, xdt):
    # decode-once path (M >= 1024) with both activation types; the workspace
    # (the decoded weight copy) starts full of garbage and is sized by the API
    M, N, K = 1100, 528, 320
    codes, scales = workloads.random_packed(N, K, "weight", seed=81)
    X = workloads.vectors(M, K, seed=82, dtype=xdt)
    need = R.razer_workspace_size(R.RAZER_OP_GEMM, M, N, K)
    assert need == N * K * 2
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=DEV)
    Y = R.razer_gemm(X.to(DEV), codes.to(DEV), scales.to(DEV), torch.tensor([0.05], device=DEV), "weight", torch.float32, workspace=ws)
    torch.cuda.synchronize()
    assert R.razer_get_device_status() == 0
    ref = orc.gemm_ref(oracle_in(X), codes.numpy(), scales.numpy(), 0.05, 0)
    assert rel_err(Y.cpu().numpy(), ref) <= REL_TOL
    # below M = 256, and below M = 1024 for weight matrices of more than 2^25
    # elements, no workspace is needed (fused decode)
    assert R.razer_workspace_size(R.RAZER_OP_GEMM, 255, N, K) == 0
    assert R.razer_workspace_size(R.RAZER_OP_GEMM, 1023, 8192, 8192) == 0
    assert R.razer_workspace_size(R.RAZER_OP_GEMM, 1023, N, K) == N * K * 2


# --- W4A4 product of two RaZeR-packed operands ------------------------------
def w4a4(ca, sa, ts_a, afmt, cw, sw, ts_w, wfmt, out_dtype=torch.float32, workspace=None):
    t = lambda v: torch.tensor([v], dtype=torch.float32, device=DEV)
    Y = R.razer_gemm_w4a4(ca.to(DEV), sa.to(DEV), t(ts_a), cw.to(DEV), sw.to(DEV), t(ts_w), afmt, wfmt, out_dtype,
                          workspace=workspace)
    torch.cuda.synchronize()
    return Y


@pytest.mark.parametrize("afmt,wfmt", [("act", "weight"), ("nvfp4", "nvfp4"), ("act", "act"), ("weight", "weight")])
def test_w4a4_random_packed(orc, afmt, wfmt):
    # ragged M and N over several 256 x 256 tiles, 5 k-steps; random packed
    # operands reach every code, meta value and subnormal scale code
    M, N, K = 300, 272, 320
    ca, sa = workloads.random_packed(M, K, afmt, seed=61, max_scale_code=60)
    cw, sw = workloads.random_packed(N, K, wfmt, seed=62, max_scale_code=60)
    ts_a, ts_w = 0.0173, 0.00311
    ref = orc.gemm_w4a4_ref(ca.numpy(), sa.numpy(), ts_a, FMT_ID[afmt], cw.numpy(), sw.numpy(), ts_w, FMT_ID[wfmt])
    Y = w4a4(ca, sa, ts_a, afmt, cw, sw, ts_w, wfmt)
    assert rel_err(Y.cpu().numpy(), ref) <= REL_TOL
    for odt in (torch.float16, torch.bfloat16):
        assert_close_typed(w4a4(ca, sa, ts_a, afmt, cw, sw, ts_w, wfmt, odt), ref)


def test_w4a4_oracle_quantized_pipeline(orc):
    # activations with outlier channels and weights, both quantized by the
    # oracle (activations: dynamic ts, E4M3 + 1-bit meta; weights: E3M3 +
    # 2-bit meta); the GPU product of the packed tensors against the oracle's
    M, N, K = 384, 512, 1024
    x = workloads.outlier_activations(M, K, seed=63)
    w = workloads.weight(N, K, std=0.02, seed=64)
    ca, sa, ts_a, _ = orc.quantize(oracle_in(x), FMT_ID["act"])
    cw, sw, ts_w, _ = orc.quantize(w.numpy(), FMT_ID["weight"])
    ref = orc.gemm_w4a4_ref(ca, sa, ts_a, FMT_ID["act"], cw, sw, ts_w, FMT_ID["weight"])
    Y = w4a4(torch.from_numpy(ca), torch.from_numpy(sa), ts_a, "act", torch.from_numpy(cw), torch.from_numpy(sw), ts_w, "weight")
    assert rel_err(Y.cpu().numpy(), ref) <= REL_TOL


@pytest.mark.parametrize("M,N,K", [(4096, 4096, 4096), (1024, 1024, 28672)])
def test_w4a4_full_size_sampled(orc, M, N, K):
    # the prefill shape and a K that runs in two accumulation chains; 24
    # sampled rows against the oracle, workspace full of garbage
    ca, sa = workloads.random_packed(M, K, "act", seed=M + 1, max_scale_code=60)
    cw, sw = workloads.random_packed(N, K, "weight", seed=N + 2, max_scale_code=40)
    ts_a, ts_w = 0.011, 0.0042
    ws = torch.full((R.razer_workspace_size(R.RAZER_OP_GEMM_W4A4, M, N, K),), 0xFF, dtype=torch.uint8, device=DEV)
    Y = w4a4(ca, sa, ts_a, "act", cw, sw, ts_w, "weight", workspace=ws).cpu().numpy()
    rows = np.random.default_rng(K).choice(M, 24, replace=False)
    ref = orc.gemm_w4a4_ref(ca.numpy(), sa.numpy(), ts_a, FMT_ID["act"], cw.numpy(), sw.numpy(), ts_w, FMT_ID["weight"], rows=rows)
    assert rel_err(Y[rows], ref) <= REL_TOL


@pytest.mark.parametrize("afmt", ["act", "nvfp4"])
@pytest.mark.parametrize("xdt", [torch.bfloat16, torch.float16])
def test_w4a4_online_equals_two_calls(orc, afmt, xdt):
    # the fused quantize + decode path gives bit for bit what
    # razer_quantize_acts followed by razer_gemm_w4a4 gives (dynamic ts, meta
    # histogram, codes kept); both against the oracle's product of the
    # oracle-quantized activations
    M, N, K = 300, 272, 512
    x = workloads.outlier_activations(M, K, seed=90, dtype=xdt)
    cw, sw = workloads.random_packed(N, K, "weight", seed=91, max_scale_code=40)
    xd, cwd, swd = x.to(DEV), cw.to(DEV), sw.to(DEV)
    tw = torch.tensor([0.0043], dtype=torch.float32, device=DEV)
    Y1, ts_a, kept, mh = R.razer_gemm_w4a4_online(xd, cwd, swd, tw, None, afmt, "weight", torch.float32, keep_codes=True,
                                                  hist=afmt == "act")
    ca, sa, t2, h2 = R.razer_quantize_acts(xd, None, afmt, hist=afmt == "act")
    Y2 = R.razer_gemm_w4a4(ca, sa, t2, cwd, swd, tw, afmt, "weight", torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2) and torch.equal(ts_a, t2)
    assert torch.equal(kept[0], ca) and torch.equal(kept[1], sa)
    if afmt == "act":
        assert torch.equal(mh, h2)
    oca, osa, ots, _ = orc.quantize(oracle_in(x), FMT_ID[afmt])
    assert float(ts_a.cpu()[0]) == ots
    ref = orc.gemm_w4a4_ref(oca, osa, ots, FMT_ID[afmt], cw.numpy(), sw.numpy(), 0.0043, FMT_ID["weight"])
    assert rel_err(Y1.cpu().numpy(), ref) <= REL_TOL


def test_w4a4_online_static_scale(orc):
    # a given activation scale (no amax pass); no codes kept, bf16 output
    M, N, K = 256, 256, 1024
    x = workloads.outlier_activations(M, K, seed=92)
    w = workloads.weight(N, K, seed=93)
    cw, sw, tw, _ = orc.quantize(w.numpy(), FMT_ID["weight"])
    ts_in = 0.0371
    oca, osa, _, _ = orc.quantize(oracle_in(x), FMT_ID["act"], ts=ts_in)
    ref = orc.gemm_w4a4_ref(oca, osa, ts_in, FMT_ID["act"], cw, sw, tw, FMT_ID["weight"])
    Y, ts_a, kept, _ = R.razer_gemm_w4a4_online(x.to(DEV), torch.from_numpy(cw).to(DEV), torch.from_numpy(sw).to(DEV),
                                                torch.tensor([tw], dtype=torch.float32, device=DEV),
                                                torch.tensor([ts_in], dtype=torch.float32, device=DEV), "act", "weight", torch.bfloat16)
    torch.cuda.synchronize()
    assert kept is None and float(ts_a.cpu()[0]) == np.float32(ts_in)
    assert_close_typed(Y, ref)
