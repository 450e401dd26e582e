"""RaZeR (Redundant Zero Remapping for NVFP4) hot path for NVIDIA B200 (sm_100a).

The compute runs in librazer.so (CUDA kernels behind the C ABI of
include/razer.h); this package is its thin Python binding plus the seeded
synthetic workload generators used by the tests and the benchmark.
"""
from .razer import (  # noqa: F401
    FORMATS, RAZER_BF16, RAZER_F16, RAZER_F32, RAZER_FMT_ACT, RAZER_FMT_NVFP4, RAZER_FMT_WEIGHT,
    RAZER_OP_GEMM, RAZER_OP_GEMV, RazerError, load, razer_dequant, razer_gemm, razer_gemv,
    razer_gemv_batch, razer_gemv_batch_workspace_size, razer_gemm_w4a4, razer_gemm_w4a4_online, RAZER_OP_GEMM_W4A4, razer_quant_error, razer_quantize_variant,
    razer_quant_error_variant, razer_dequant_variant, razer_gemv_variant, razer_gemm_variant, RAZER_OP_GEMM_VARIANT,
    RAZER_FMT_FOUR_OVER_SIX, RAZER_SCALE_F16,
    razer_get_device_status, razer_quantize_acts, razer_quantize_weights, razer_quantize_weights_batch,
    razer_status_string,
    razer_version, razer_workspace_size, razer_debug_set_fault_injection, razer_set_quantize_path,
)
