"""razer_gemv_noalloc: the GEMV entry point for callers that cannot allocate
device memory (a runtime that keeps all GPU memory in its own pool, or a
fixed static memory budget, leaves them unable to pass razer_gemv a
workspace).  It must agree with razer_gemv; called through the C ABI twice in
a row, since the second call finds the first call's partials in the shared
scratch array.  This file is collected last on purpose."""
import ctypes

import pytest
import torch

import bit_quantization_razer_b200 as R
from bit_quantization_razer_b200 import workloads
from tests.gpu_helpers import REL_TOL, cuda, rel_err

pytestmark = [pytest.mark.gpu, cuda]
DEV = "cuda:0"


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_gemv_noalloc_matches_gemv_on_two_calls():
    L = R.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [(4096, 4096, 4, "weight", torch.float16, 501), (1000, 2048, 17, "act", torch.bfloat16, 502)]
    for N, K, B, fmt, xdt, seed in cases:
        codes, scales = workloads.random_packed(N, K, fmt, seed=seed, max_scale_code=40)
        codes, scales = codes.to(DEV), scales.to(DEV)
        x = workloads.vectors(B, K, seed=seed + 1, dtype=xdt).to(DEV)
        ts = torch.tensor([0.0371], dtype=torch.float32, device=DEV)
        assert R.razer_workspace_size(R.RAZER_OP_GEMV, B, N, K) <= L.razer_gemv_noalloc_max_scratch()
        ref = R.razer_gemv(x, codes, scales, ts, fmt, torch.float32)
        out = torch.full((B, N), float("nan"), dtype=torch.float32, device=DEV)
        st = L.razer_gemv_noalloc(_ptr(x), R.RAZER_F16 if xdt == torch.float16 else R.RAZER_BF16, B, _ptr(codes),
                                  _ptr(scales), _ptr(ts), R.FORMATS[fmt], N, K, _ptr(out), R.RAZER_F32, stream)
        assert st == 0, R.razer_status_string(st)
        torch.cuda.synchronize()
        assert rel_err(out.cpu().numpy(), ref.cpu().numpy()) <= REL_TOL


def test_gemv_noalloc_rejects_sizes_beyond_the_scratch():
    L = R.load()
    B, N, K = 32, 100000, 128
    assert R.razer_workspace_size(R.RAZER_OP_GEMV, B, N, K) > L.razer_gemv_noalloc_max_scratch()
    fake = ctypes.c_void_p(0x1000)  # rejected before any device access
    st = L.razer_gemv_noalloc(fake, R.RAZER_F16, B, fake, fake, fake, R.RAZER_FMT_WEIGHT, N, K, fake, R.RAZER_F32, None)
    assert st == 5  # RAZER_ERR_WORKSPACE
