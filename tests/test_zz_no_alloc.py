"""razer_gemv_noalloc: the GEMV entry point for callers that cannot allocate
device memory (a runtime that keeps all GPU memory in its own pool, or a
fixed static memory budget, leaves them unable to pass razer_gemv a
workspace).  Called through the C ABI and checked against the oracle's
double-accumulated product and against razer_gemv, on back-to-back calls:
the second call of a shape finds the first call's partials in the shared
scratch array and must not be affected by them.  This file is collected last
on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantization_razer_b200 as R
from bit_quantization_razer_b200 import workloads
from tests.gpu_helpers import FMT_ID, REL_TOL, cuda, oracle_in, rel_err

pytestmark = [pytest.mark.gpu, cuda]
DEV = "cuda:0"


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _noalloc(x, codes, scales, ts, fmt, N, K, out):
    L = R.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    B = x.shape[0]
    xdt = R.RAZER_F16 if x.dtype == torch.float16 else R.RAZER_BF16
    st = L.razer_gemv_noalloc(_ptr(x), xdt, B, _ptr(codes), _ptr(scales), _ptr(ts), R.FORMATS[fmt], N, K, _ptr(out),
                              R.RAZER_F32, stream)
    assert st == 0, R.razer_status_string(st)
    torch.cuda.synchronize()


@pytest.mark.parametrize("N,K,B,fmt,xdt", [(4096, 4096, 4, "weight", torch.float16), (4096, 4096, 1, "weight", torch.float16),
                                           (1000, 2048, 17, "act", torch.bfloat16), (300, 1152, 3, "nvfp4", torch.float16)])
def test_gemv_noalloc_two_calls_against_oracle_and_gemv(orc, N, K, B, fmt, xdt):
    L = R.load()
    assert R.razer_workspace_size(R.RAZER_OP_GEMV, B, N, K) <= L.razer_gemv_noalloc_max_scratch()
    # two calls in a row with the same shape and different inputs
    for call in range(2):
        seed = 500 + 10 * call + B
        codes, scales = workloads.random_packed(N, K, fmt, seed=seed, max_scale_code=40)
        x = workloads.vectors(B, K, seed=seed + 1, dtype=xdt)
        ts_v = 0.0371 * (1 + call)
        codes_d, scales_d, x_d = codes.to(DEV), scales.to(DEV), x.to(DEV)
        ts = torch.tensor([ts_v], dtype=torch.float32, device=DEV)
        out = torch.full((B, N), float("nan"), dtype=torch.float32, device=DEV)
        _noalloc(x_d, codes_d, scales_d, ts, fmt, N, K, out)
        y = out.cpu().numpy()
        assert not np.isnan(y).any()  # every output element written
        rows = np.arange(N) if N <= 1024 else np.random.default_rng(call).choice(N, 512, replace=False)
        ref = orc.gemm_ref(oracle_in(x), codes.numpy()[rows], scales.numpy()[rows], ts_v, FMT_ID[fmt])
        assert rel_err(y[:, rows], ref) <= REL_TOL
        # and the workspace path on the same inputs
        yg = R.razer_gemv(x_d, codes_d, scales_d, ts, fmt, torch.float32).cpu().numpy()
        assert rel_err(y, yg.astype(np.float64)) <= REL_TOL


def test_gemv_noalloc_empty_shapes():
    L = R.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ts = torch.ones(1, device=DEV)
    # K = 0: empty sums, y = 0 (y starts as NaN)
    out = torch.full((3, 50), float("nan"), dtype=torch.float32, device=DEV)
    st = L.razer_gemv_noalloc(None, R.RAZER_F16, 3, None, None, _ptr(ts), R.RAZER_FMT_WEIGHT, 50, 0, _ptr(out), R.RAZER_F32, stream)
    assert st == 0, R.razer_status_string(st)
    torch.cuda.synchronize()
    assert torch.equal(out, torch.zeros_like(out))
    # N = 0: nothing to write, null output allowed
    x = torch.ones(2, 256, dtype=torch.float16, device=DEV)
    st = L.razer_gemv_noalloc(_ptr(x), R.RAZER_F16, 2, None, None, _ptr(ts), R.RAZER_FMT_WEIGHT, 0, 256, None, R.RAZER_F32, stream)
    assert st == 0, R.razer_status_string(st)


def test_gemv_noalloc_rejects_sizes_beyond_the_scratch():
    L = R.load()
    B, N, K = 32, 100000, 128
    assert R.razer_workspace_size(R.RAZER_OP_GEMV, B, N, K) > L.razer_gemv_noalloc_max_scratch()
    fake = ctypes.c_void_p(0x1000)  # rejected before any device access
    st = L.razer_gemv_noalloc(fake, R.RAZER_F16, B, fake, fake, fake, R.RAZER_FMT_WEIGHT, N, K, fake, R.RAZER_F32, None)
    assert st == 5  # RAZER_ERR_WORKSPACE
