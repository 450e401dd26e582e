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


@pytest.mark.parametrize("N,K,B", [(4096, 4096, 1), (4096, 4096, 4), (14336, 4096, 16), (4096, 14336, 1),
                                   (4096, 14336, 16), (8192, 8192, 32)])
def test_gemv_config_shapes(orc, N, K, B):
    codes, scales = workloads.random_packed(N, K, "weight", seed=N + K + B, max_scale_code=40)
    x = workloads.vectors(B, K, seed=B)
    ts = 0.0045
    y = gemv(x, codes, scales, ts, "weight").cpu().numpy()
    cols = np.random.default_rng(1).choice(N, 512, replace=False)
    ref = orc.gemm_ref(x.numpy(), codes[cols].numpy(), scales[cols].numpy(), ts, 0)
    assert rel_err(y[:, cols], ref) <= REL_TOL


def test_gemv_k128_single_chunk(orc):
    codes, scales = workloads.random_packed(48, 128, "act", seed=60)
    x = workloads.vectors(2, 128, seed=61)
    ref = orc.gemm_ref(x.numpy(), codes.numpy(), scales.numpy(), 1.5, 1)
    y = gemv(x, codes, scales, 1.5, "act").cpu().numpy()
    assert rel_err(y, ref) <= REL_TOL


def test_gemv_workspace_errors():
    codes, scales = workloads.random_packed(64, 256, "weight", seed=62)
    x = torch.ones(4, 256, dtype=torch.float16, device=DEV)
    ts = torch.ones(1, device=DEV)
    need = R.razer_workspace_size(R.RAZER_OP_GEMV, 4, 64, 256)
    small = torch.empty(max(need - 16, 16), dtype=torch.uint8, device=DEV)
    with pytest.raises(R.RazerError) as e:
        R.razer_gemv(x, codes.to(DEV), scales.to(DEV), ts, "weight", workspace=small)
    assert "WORKSPACE" in str(e.value)
