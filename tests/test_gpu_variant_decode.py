"""GPU decoder and W4A16 GEMV of the format variants against the oracle:
bit-exact decode, and products within the fp32-accumulation tolerance, for
blocks of 16-128, caller-chosen special values and the pages' kernel format
(blocks of 128, FP16 scale words with the meta in bits 15..14)."""
import numpy as np
import pytest
import torch

import bit_quantization_razer_b200 as R
from bit_quantization_razer_b200 import workloads
from tests.gpu_helpers import FMT_ID, assert_close_typed, cuda, oracle_in, rel_err, REL_TOL

pytestmark = [pytest.mark.gpu, cuda]
DEV = "cuda:0"

VARIANTS = [
    (16, "weight", [5.0, -5.0, 7.0, -7.0]),      # a per-model pair at the hot-path block
    (16, "weight", [5.0, -5.0, 9.5, -9.5]),
    (32, "weight", [2.5, -2.5, 5.0, -5.0]),
    (64, "act", [5.0, -5.0]),
    (128, "act", [4.5, -4.5]),
    (64, "nvfp4", []),
    (128, "f16_scale", [5.0, -5.0, 8.0, -8.0]),  # the pages' kernel format
    (128, "f16_scale", [2.5, -3.5, 9.5, -8.5]),
    (128, "f16_scale", []),
]
IDS = [f"b{b}-{f}-{'_'.join(str(v) for v in V) or 'plain'}" for b, f, V in VARIANTS]


def _dev(*ts):
    return [t.to(DEV) if isinstance(t, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(t)).to(DEV) for t in ts]


def _ts(v):
    return torch.tensor([v], dtype=torch.float32, device=DEV)


def _quantized(orc, N, K, block, fmt, V, seed):
    w = workloads.weight(N, K, std=0.02, seed=seed, dtype=torch.float32)
    w[1] = 0.0          # an all-zero row: scale 0 in every block
    w[2] *= 1e-3
    w = w.to(torch.float16)
    return orc.quantize_generic(w.numpy(), block, FMT_ID[fmt], V)


@pytest.mark.parametrize("block,fmt,V", VARIANTS, ids=IDS)
def test_dequant_variant_bit_exact(orc, block, fmt, V):
    codes, scales, ts = _quantized(orc, 72, 512, block, fmt, V, seed=90)
    c, s = _dev(codes, scales)
    for odt, name in ((torch.float32, "f32"), (torch.float16, "f16"), (torch.bfloat16, "bf16")):
        got = R.razer_dequant_variant(c, s, _ts(ts), block, fmt, V, odt)
        ref = orc.dequant_generic(codes, scales, ts, block, FMT_ID[fmt], V, name)
        g = got.cpu()
        g = g.numpy() if odt == torch.float32 else g.view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(g, ref)


@pytest.mark.parametrize("block,fmt,V", VARIANTS, ids=IDS)
def test_dequant_variant_random_packed(orc, block, fmt, V):
    # every code under every scale magnitude and meta value
    codes, scales = workloads.random_packed_variant(40, 1024, block, fmt, len(V), seed=91)
    ts = 0.0371
    got = R.razer_dequant_variant(*_dev(codes, scales), _ts(ts), block, fmt, V, torch.float32)
    ref = orc.dequant_generic(codes.numpy(), scales.numpy(), ts, block, FMT_ID[fmt], V, "f32")
    np.testing.assert_array_equal(got.cpu().numpy(), ref)


@pytest.mark.parametrize("B", [1, 5, 16, 32])
@pytest.mark.parametrize("block,fmt,V", VARIANTS, ids=IDS)
def test_gemv_variant_quantized(orc, block, fmt, V, B):
    # N = 200 (ragged against 16-row warps and 4-warp CTAs), K = 384 (three
    # 128-k slices, an odd count)
    N, K = 200, 384
    codes, scales, ts = _quantized(orc, N, K, block, fmt, V, seed=92)
    x = workloads.vectors(B, K, seed=93)
    y = R.razer_gemv_variant(x.to(DEV), *_dev(codes, scales), _ts(ts), block, fmt, V)
    r = orc.gemv_generic(x.numpy(), codes, scales, ts, block, FMT_ID[fmt], V)
    assert rel_err(y.cpu().numpy(), r) <= REL_TOL


@pytest.mark.parametrize("out_dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("xdt", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("block,fmt,V", [VARIANTS[0], VARIANTS[3], VARIANTS[6], VARIANTS[7]], ids=[IDS[0], IDS[3], IDS[6], IDS[7]])
def test_gemv_variant_types(orc, block, fmt, V, xdt, out_dtype):
    if xdt == torch.bfloat16 and fmt != "f16_scale" and any(abs(v) == 9.5 for v in V):
        pytest.skip("refused combination (tested separately)")
    N, K = 96, 1024
    codes, scales = workloads.random_packed_variant(N, K, block, fmt, len(V), seed=94)
    ts = 0.0193 if fmt != "f16_scale" else 1.0
    x = workloads.vectors(7, K, seed=95, dtype=xdt)
    y = R.razer_gemv_variant(x.to(DEV), *_dev(codes, scales), _ts(ts), block, fmt, V, out_dtype)
    r = orc.gemv_generic(oracle_in(x), codes.numpy(), scales.numpy(), ts, block, FMT_ID[fmt], V)
    assert_close_typed(y, r)


def test_gemv_variant_bf16_with_eight_and_a_half(orc):
    # 8.5 times every scale significand fits bf16's 8 bits: allowed and exact
    N, K = 80, 512
    V = [5.0, -5.0, 8.5, -8.5]
    codes, scales = workloads.random_packed_variant(N, K, 16, "weight", 4, seed=103)
    x = workloads.vectors(3, K, seed=104, dtype=torch.bfloat16)
    y = R.razer_gemv_variant(x.to(DEV), *_dev(codes, scales), _ts(0.0625), 16, "weight", V)
    r = orc.gemv_generic(oracle_in(x), codes.numpy(), scales.numpy(), 0.0625, 16, 0, V)
    assert rel_err(y.cpu().numpy(), r) <= REL_TOL


def test_gemv_variant_bf16_with_nine_and_a_half_is_refused():
    codes, scales = workloads.random_packed_variant(16, 128, 16, "weight", 4, seed=96)
    x = workloads.vectors(1, 128, seed=97, dtype=torch.bfloat16)
    with pytest.raises(R.RazerError):
        R.razer_gemv_variant(x.to(DEV), *_dev(codes, scales), _ts(1.0), 16, "weight", [5.0, -5.0, 9.5, -9.5])


def test_gemv_variant_block16_matches_product_reference(orc):
    # block 16 with the weight format's own values is the hot-path format:
    # the variant kernel agrees with the pinned product reference
    N, K = 128, 512
    w = workloads.weight(N, K, seed=98)
    codes, scales, ts, _ = orc.quantize(w.numpy(), 0)
    x = workloads.vectors(3, K, seed=99)
    y = R.razer_gemv_variant(x.to(DEV), *_dev(codes, scales), _ts(ts), 16, "weight", [5.0, -5.0, 8.0, -8.0])
    assert rel_err(y.cpu().numpy(), orc.gemm_ref(x.numpy(), codes, scales, ts, 0)) <= REL_TOL


@pytest.mark.parametrize("B", [1, 16])
@pytest.mark.parametrize("fmt,block,V", [("f16_scale", 128, [5.0, -5.0, 8.0, -8.0]), ("weight", 16, [5.0, -5.0, 7.0, -7.0])])
def test_gemv_variant_full_size_sampled(orc, fmt, block, V, B):
    # the Llama-3-8B MLP up-projection shape, random packed weights; sampled
    # output rows against the oracle
    N, K = 14336, 4096
    codes, scales = workloads.random_packed_variant(N, K, block, fmt, len(V), seed=100)
    ts = 1.0 if fmt == "f16_scale" else 2.0 ** -9
    x = workloads.vectors(B, K, seed=101)
    y = R.razer_gemv_variant(x.to(DEV), *_dev(codes, scales), _ts(ts), block, fmt, V).cpu().numpy()
    rows = np.sort(np.random.default_rng(102).choice(N, 48, replace=False))
    rows = np.concatenate([rows, [0, N - 1]])
    r = orc.gemv_generic(x.numpy(), codes.numpy()[rows], scales.numpy()[rows], ts, block, FMT_ID[fmt], V)
    assert rel_err(y[:, rows], r) <= REL_TOL


def test_gemv_variant_empty_and_zero_k():
    codes = torch.zeros((0, 64), dtype=torch.uint8, device=DEV)
    scales = torch.zeros((0, 2), dtype=torch.uint8, device=DEV)
    x = torch.randn(2, 128, device=DEV).half()
    y = R.razer_gemv_variant(x, codes, scales, _ts(1.0), 128, "f16_scale", [5.0, -5.0])
    assert y.shape == (2, 0)
    c0 = torch.zeros((8, 0), dtype=torch.uint8, device=DEV)
    s0 = torch.zeros((8, 0), dtype=torch.uint8, device=DEV)
    x0 = torch.zeros((2, 0), device=DEV).half()
    y0 = R.razer_gemv_variant(x0, c0, s0, _ts(1.0), 128, "f16_scale", [5.0, -5.0], out=torch.full((2, 8), 7.0, device=DEV))
    torch.cuda.synchronize()
    assert not y0.any()


# --- prefill GEMM on variant weights -----------------------------------------
@pytest.mark.parametrize("M", [64, 300])
@pytest.mark.parametrize("block,fmt,V", VARIANTS, ids=IDS)
def test_gemm_variant_quantized(orc, block, fmt, V, M):
    # oracle-quantized weights (zero and tiny rows), ragged N and M tiles
    N, K = 200, 384
    codes, scales, ts = _quantized(orc, N, K, block, fmt, V, seed=92)
    X = workloads.vectors(M, K, seed=110)
    Y = R.razer_gemm_variant(X.to(DEV), *_dev(codes, scales), _ts(ts), block, fmt, V, torch.float32)
    r = orc.gemv_generic(X.numpy(), codes, scales, ts, block, FMT_ID[fmt], V)
    assert rel_err(Y.cpu().numpy(), r) <= REL_TOL


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("block,fmt,V", [VARIANTS[0], VARIANTS[2], VARIANTS[3], VARIANTS[5], VARIANTS[6], VARIANTS[7]],
                         ids=[IDS[0], IDS[2], IDS[3], IDS[5], IDS[6], IDS[7]])
def test_gemm_variant_bf16_random_packed(orc, block, fmt, V, out_dtype):
    # bf16 activations (the weight copy is bf16: exact without +-9.5; FP16
    # scale words as two exact bf16 terms), every code under every scale
    # magnitude, K spanning several k-steps
    M, N, K = 320, 96, 1024
    codes, scales = workloads.random_packed_variant(N, K, block, fmt, len(V), seed=111)
    X = workloads.vectors(M, K, seed=112, dtype=torch.bfloat16)
    Y = R.razer_gemm_variant(X.to(DEV), *_dev(codes, scales), _ts(0.0193), block, fmt, V, out_dtype)
    r = orc.gemv_generic(oracle_in(X), codes.numpy(), scales.numpy(), 0.0193, block, FMT_ID[fmt], V)
    assert_close_typed(Y, r)


def test_gemm_variant_refusals():
    codes, scales = workloads.random_packed_variant(16, 256, 16, "weight", 4, seed=113)
    X = workloads.vectors(8, 256, seed=114, dtype=torch.bfloat16)
    with pytest.raises(R.RazerError):  # bf16 cannot hold 9.5 x every scale
        R.razer_gemm_variant(X.to(DEV), *_dev(codes, scales), _ts(1.0), 16, "weight", [5.0, -5.0, 9.5, -9.5])
    c2, s2 = workloads.random_packed_variant(16, 96, 32, "f16_scale", 4, seed=115)
    with pytest.raises(R.RazerError):  # FP16 scale words need whole 64-element k-steps
        R.razer_gemm_variant(workloads.vectors(8, 96).to(DEV), *_dev(c2, s2), _ts(1.0), 32, "f16_scale", [5.0, -5.0, 8.0, -8.0])
    with pytest.raises(R.RazerError):  # K not a multiple of the block
        R.razer_gemm_variant(workloads.vectors(8, 96).to(DEV), *_dev(c2, s2), _ts(1.0), 64, "f16_scale", [5.0])


@pytest.mark.parametrize("M", [100, 1100])
def test_gemm_variant_hot_path_format_equals_razer_gemm(M):
    # block 16, E3M3 scales, V = +-5/+-8 is the hot-path weight format: the
    # variant GEMM's exact q*s copy and razer_gemm's q*s*2^-8 copy differ by a
    # power of two that the epilogue undoes exactly, so the outputs are equal
    N, K = 272, 640
    codes, scales = workloads.random_packed(N, K, "weight", seed=116, max_scale_code=40)
    X = workloads.vectors(M, K, seed=117, dtype=torch.bfloat16).to(DEV)
    c, s = _dev(codes, scales)
    a = R.razer_gemm_variant(X, c, s, _ts(0.037), 16, "weight", [5.0, -5.0, 8.0, -8.0], torch.float32)
    b = R.razer_gemm(X, c, s, _ts(0.037), "weight", torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(a.cpu().numpy(), b.cpu().numpy())


def test_gemm_variant_pages_format_sampled(orc):
    # the pages' kernel format (blocks of 128, FP16 scale words, +-5/+-8) on a
    # prefill shape, fp16 activations; sampled rows against the oracle
    M, N, K = 2048, 4096, 4096
    codes, scales = workloads.random_packed_variant(N, K, 128, "f16_scale", 4, seed=118)
    X = workloads.vectors(M, K, seed=119)
    Y = R.razer_gemm_variant(X.to(DEV), *_dev(codes, scales), _ts(1.0), 128, "f16_scale", [5.0, -5.0, 8.0, -8.0],
                             torch.float32).cpu().numpy()
    rows = np.sort(np.random.default_rng(120).choice(M, 24, replace=False))
    r = orc.gemv_generic(X.numpy()[rows], codes.numpy(), scales.numpy(), 1.0, 128, FMT_ID["f16_scale"], [5.0, -5.0, 8.0, -8.0])
    assert rel_err(Y[rows], r) <= REL_TOL


def test_gemm_variant_empty_shapes():
    c, s = workloads.random_packed_variant(8, 128, 128, "f16_scale", 2, seed=121)
    X0 = torch.zeros((0, 128), device=DEV).half()
    Y0 = R.razer_gemm_variant(X0, *_dev(c, s), _ts(1.0), 128, "f16_scale", [5.0, -5.0], torch.float32)
    assert Y0.shape == (0, 8)
    c0 = torch.zeros((8, 0), dtype=torch.uint8, device=DEV)
    s0 = torch.zeros((8, 0), dtype=torch.uint8, device=DEV)
    X = torch.zeros((3, 0), device=DEV).half()
    Y = R.razer_gemm_variant(X, c0, s0, _ts(1.0), 128, "f16_scale", [5.0, -5.0], torch.float32,
                             out=torch.full((3, 8), 7.0, device=DEV))
    torch.cuda.synchronize()
    assert not Y.any()
