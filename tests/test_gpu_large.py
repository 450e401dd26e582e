"""Parity at sizes past 2^31 elements (64-bit indexing in every kernel).

Inputs are drawn on the device by torch's seeded generator (a stand-in for
the host generator that would take minutes at these sizes); sampled rows,
including the last ones, are compared with the oracle."""
import numpy as np
import pytest
import torch

import bit_quantization_razer_b200 as R
from tests.gpu_helpers import assert_close_typed, cuda, rel_err, REL_TOL

pytestmark = [pytest.mark.gpu, cuda]
DEV = "cuda:0"


def _normal_fp16(rows, cols, std, seed, chunk=2048):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    out = torch.empty((rows, cols), dtype=torch.float16, device=DEV)
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        out[r0:r1] = (torch.randn((r1 - r0, cols), generator=g, device=DEV) * std).half()
    # 0.1% of the entries x10 (the weight recipe's outliers)
    flat = out.view(-1)
    idx = torch.randint(0, flat.numel(), (flat.numel() // 1000,), generator=g, device=DEV)
    flat[idx] = (flat[idx].float() * 10).half()
    return out


def _random_packed_device(N, K, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    codes = torch.randint(0, 256, (N, K // 2), generator=g, device=DEV, dtype=torch.int32).to(torch.uint8)
    mag = torch.randint(0, 41, (N, K // 16), generator=g, device=DEV, dtype=torch.int32)
    meta = torch.randint(0, 4, (N, K // 16), generator=g, device=DEV, dtype=torch.int32)
    return codes, (mag | (meta << 6)).to(torch.uint8)


def test_quantize_past_2pow31_elements(orc):
    Rr, K = 16400, 131072  # 2 149 580 800 elements, 4.3 GB of fp16
    assert Rr * K > 2 ** 31
    W = _normal_fp16(Rr, K, 0.02, seed=200)
    c, s, t = R.razer_quantize_weights(W)
    torch.cuda.synchronize()
    assert R.razer_get_device_status() == 0
    ts = orc.tensor_scale(W.cpu().numpy(), 0)
    assert float(t.cpu()[0]) == ts
    rows = [0, 1, Rr // 2, Rr - 2, Rr - 1]
    oc, os_, _, _ = orc.quantize(W[rows].cpu().numpy(), 0, ts=ts)
    np.testing.assert_array_equal(c[rows].cpu().numpy(), oc)
    np.testing.assert_array_equal(s[rows].cpu().numpy(), os_)
    del W, c, s


@pytest.mark.parametrize("B", [1, 16])
def test_gemv_codes_past_2pow31_bytes(orc, B):
    N, K = 131072, 32768  # codes 2 GiB + scales 256 MiB
    assert N * K // 2 >= 2 ** 31
    codes, scales = _random_packed_device(N, K, seed=201)
    g = torch.Generator(device=DEV)
    g.manual_seed(202)
    x = torch.randn((B, K), generator=g, device=DEV).half()
    ts = torch.tensor([2.0 ** -9], dtype=torch.float32, device=DEV)
    y = R.razer_gemv(x, codes, scales, ts, "weight", torch.float32)
    torch.cuda.synchronize()
    rows = [0, 127, N // 2 + 5, N - 129, N - 1]
    r = orc.gemm_ref(x.cpu().numpy(), codes[rows].cpu().numpy(), scales[rows].cpu().numpy(), 2.0 ** -9, 0)
    assert rel_err(y[:, rows].cpu().numpy(), r) <= REL_TOL
    del codes, scales


def test_gemm_output_past_2pow31_elements(orc):
    M, N, K = 8192, 262400, 256  # Y: 2 149 580 800 bf16 elements
    assert M * N > 2 ** 31
    codes, scales = _random_packed_device(N, K, seed=203)
    g = torch.Generator(device=DEV)
    g.manual_seed(204)
    X = torch.randn((M, K), generator=g, device=DEV).to(torch.bfloat16)
    ts = torch.tensor([2.0 ** -9], dtype=torch.float32, device=DEV)
    Y = R.razer_gemm(X, codes, scales, ts, "weight", torch.bfloat16)
    torch.cuda.synchronize()
    assert R.razer_get_device_status() == 0
    rows = [0, M // 2 + 3, M - 1]
    from tests.gpu_helpers import oracle_in
    r = orc.gemm_ref(oracle_in(X[rows]), codes.cpu().numpy(), scales.cpu().numpy(), 2.0 ** -9, 0)
    assert_close_typed(Y[rows], r)
    del Y, codes, scales
