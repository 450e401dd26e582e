"""Shared helpers of the GPU parity tests (oracle adapters and tolerances)."""
import numpy as np
import pytest
import torch

from bit_quantization_razer_b200 import workloads

cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

FMT_ID = {"weight": 0, "act": 1, "nvfp4": 2, "f16_scale": 4}

# Tolerance of the products (fp32 accumulation against the oracle's double
# accumulation): max |y - r| / max(|r|, 0.01 * rms(r)) <= 2e-3.
REL_TOL = 2e-3


def oracle_in(t: torch.Tensor):
    import oracle

    t = t.cpu()
    if t.dtype == torch.bfloat16:
        return oracle.Bf16Bits(workloads.to_numpy_bits(t))
    return t.numpy()


def rel_err(y: np.ndarray, r: np.ndarray) -> float:
    y = np.asarray(y, np.float64)
    r = np.asarray(r, np.float64)
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    floor = max(0.01 * rms, 1e-30)
    return float(np.max(np.abs(y - r) / np.maximum(np.abs(r), floor))) if r.size else 0.0


def half_ulp(r: np.ndarray, dtype) -> np.ndarray:
    """Half a unit in the last place of |r| in an fp16/bf16 output type."""
    a = np.abs(r).astype(np.float64)
    if dtype == torch.float16:
        e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
        return 0.5 * 2.0 ** (e - 10)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 0.5 * 2.0 ** (e - 7)


def assert_close_typed(y: torch.Tensor, r: np.ndarray):
    yv = y.float().cpu().numpy().astype(np.float64)
    if y.dtype == torch.float32:
        assert rel_err(yv, r) <= REL_TOL
        return
    rms = float(np.sqrt(np.mean(r * r)))
    bound = REL_TOL * np.maximum(np.abs(r), 0.01 * rms) + half_ulp(r, y.dtype)
    assert np.all(np.abs(yv - r) <= bound)
