"""ctypes binding of librazer.so (declared in include/razer.h).

Argument marshalling only: every step of the RaZeR path runs in the CUDA
kernels of the library.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing or a call fails,
an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librazer.so")

# enums of include/razer.h
RAZER_OK = 0
STATUS_NAMES = {
    0: "RAZER_OK", 1: "RAZER_ERR_INVALID_ARG", 2: "RAZER_ERR_SHAPE", 3: "RAZER_ERR_ALIGN",
    4: "RAZER_ERR_DTYPE", 5: "RAZER_ERR_WORKSPACE", 6: "RAZER_ERR_UNSUPPORTED",
    7: "RAZER_ERR_TIMEOUT", 8: "RAZER_ERR_CUDA",
}
RAZER_F16, RAZER_BF16, RAZER_F32 = 0, 1, 2
RAZER_FMT_WEIGHT, RAZER_FMT_ACT, RAZER_FMT_NVFP4, RAZER_FMT_FOUR_OVER_SIX, RAZER_SCALE_F16 = 0, 1, 2, 3, 4
RAZER_OP_GEMV, RAZER_OP_GEMM, RAZER_OP_GEMM_W4A4, RAZER_OP_GEMM_VARIANT = 0, 1, 2, 3
FORMATS = {"weight": RAZER_FMT_WEIGHT, "act": RAZER_FMT_ACT, "nvfp4": RAZER_FMT_NVFP4, "four_over_six": RAZER_FMT_FOUR_OVER_SIX,
           "f16_scale": RAZER_SCALE_F16}
_DT = {torch.float16: RAZER_F16, torch.bfloat16: RAZER_BF16, torch.float32: RAZER_F32}

EXPORTED = (
    "razer_quantize_weights", "razer_quantize_weights_batch", "razer_quantize_acts", "razer_dequant", "razer_gemv", "razer_gemm",
    "razer_gemv_batch", "razer_gemv_batch_workspace_size", "razer_gemm_w4a4", "razer_gemm_w4a4_online", "razer_quant_error",
    "razer_quantize_variant", "razer_quant_error_variant", "razer_dequant_variant", "razer_gemv_variant", "razer_gemm_variant",
    "razer_workspace_size", "razer_get_device_status", "razer_status_string", "razer_version",
    "razer_gemv_noalloc", "razer_gemv_noalloc_max_scratch", "razer_debug_set_fault_injection", "razer_set_quantize_path",
)


class GemvProblem(ctypes.Structure):
    """razer_gemv_problem of include/razer.h."""
    _fields_ = [("x", ctypes.c_void_p), ("B", ctypes.c_int64), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("ts", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("y", ctypes.c_void_p)]


class RazerError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


_lib = None


def load() -> ctypes.CDLL:
    """Load librazer.so (built in-tree by bit_quantization_razer_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: run `python -m bit_quantization_razer_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    L.razer_quantize_weights.argtypes = [vp, i32, i64, i64, vp, vp, vp, i32, vp]
    L.razer_quantize_weights_batch.argtypes = [i32, ctypes.POINTER(vp), i32, ctypes.POINTER(i64), ctypes.POINTER(i64),
                                               ctypes.POINTER(vp), ctypes.POINTER(vp), vp, i32, vp]
    L.razer_quantize_acts.argtypes = [vp, i32, i64, i64, vp, vp, vp, vp, vp, i32, vp]
    L.razer_dequant.argtypes = [vp, vp, vp, i32, i64, i64, vp, i32, vp]
    L.razer_gemv.argtypes = [vp, i32, i64, vp, vp, vp, i32, i64, i64, vp, i32, vp, sz, vp]
    L.razer_gemm.argtypes = [vp, i32, i64, vp, vp, vp, i32, i64, i64, vp, i32, vp, sz, vp]
    L.razer_gemv_batch.argtypes = [i32, ctypes.POINTER(GemvProblem), i32, i32, i32, vp, sz, vp]
    L.razer_gemm_w4a4.argtypes = [vp, vp, vp, i32, i64, vp, vp, vp, i32, i64, i64, vp, i32, vp, sz, vp]
    L.razer_gemm_w4a4_online.argtypes = [vp, i32, i64, vp, i32, vp, vp, vp, vp, vp, vp, vp, i32, i64, i64, vp, i32, vp, sz, vp]
    L.razer_quantize_variant.argtypes = [vp, i32, i64, i64, i32, i32, ctypes.POINTER(ctypes.c_float), i32, vp, vp, vp, vp]
    L.razer_quant_error_variant.argtypes = [vp, i32, i64, i64, i32, i32, ctypes.POINTER(ctypes.c_float), i32, vp, vp, vp, vp, vp]
    L.razer_dequant_variant.argtypes = [vp, vp, vp, i64, i64, i32, i32, ctypes.POINTER(ctypes.c_float), i32, vp, i32, vp]
    L.razer_gemv_variant.argtypes = [vp, i32, i64, vp, vp, vp, i32, i32, ctypes.POINTER(ctypes.c_float), i32, i64, i64, vp, i32, vp,
                                     sz, vp]
    L.razer_gemm_variant.argtypes = [vp, i32, i64, vp, vp, vp, i32, i32, ctypes.POINTER(ctypes.c_float), i32, i64, i64, vp, i32, vp,
                                     sz, vp]
    L.razer_quant_error.argtypes = [vp, i32, i64, i64, vp, vp, vp, i32, vp, vp]
    L.razer_gemv_batch_workspace_size.argtypes = [i32, ctypes.POINTER(GemvProblem)]
    L.razer_gemv_batch_workspace_size.restype = sz
    L.razer_gemv_noalloc.argtypes = [vp, i32, i64, vp, vp, vp, i32, i64, i64, vp, i32, vp]
    L.razer_gemv_noalloc.restype = ctypes.c_int
    L.razer_gemv_noalloc_max_scratch.argtypes = []
    L.razer_gemv_noalloc_max_scratch.restype = sz
    L.razer_workspace_size.argtypes = [i32, i64, i64, i64]
    L.razer_workspace_size.restype = sz
    L.razer_get_device_status.argtypes = [vp]
    L.razer_status_string.argtypes = [i32]
    L.razer_status_string.restype = ctypes.c_char_p
    L.razer_version.argtypes = []
    L.razer_debug_set_fault_injection.argtypes = [i32]
    L.razer_debug_set_fault_injection.restype = ctypes.c_int
    L.razer_set_quantize_path.argtypes = [i32]
    L.razer_set_quantize_path.restype = ctypes.c_int
    for fn in ("razer_quantize_variant", "razer_quant_error_variant", "razer_dequant_variant", "razer_gemv_variant", "razer_gemm_variant",
               "razer_gemm_w4a4_online", "razer_quant_error", "razer_gemm_w4a4", "razer_gemv_batch", "razer_quantize_weights", "razer_quantize_weights_batch", "razer_quantize_acts", "razer_dequant", "razer_gemv", "razer_gemm",
               "razer_get_device_status", "razer_version"):
        getattr(L, fn).restype = ctypes.c_int
    _lib = L
    return L


def _p(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, status: int):
    if status != RAZER_OK:
        raise RazerError(fn, status)


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def razer_quantize_weights(W: torch.Tensor, fmt="weight", *, codes=None, scales=None, ts=None, stream=None):
    """Quantize W [N, K] (fp16/bf16, CUDA). Returns (codes [N, K/2] u8,
    scales [N, K/16] u8, ts [1] f32), all on W's device."""
    N, K = W.shape
    dev = W.device
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev) if codes is None else codes
    scales = torch.empty((N, K // 16), dtype=torch.uint8, device=dev) if scales is None else scales
    ts = torch.empty(1, dtype=torch.float32, device=dev) if ts is None else ts
    st = load().razer_quantize_weights(_p(W), _DT.get(W.dtype, -1), N, K, _p(codes), _p(scales), _p(ts), _fmt(fmt), _stream(stream))
    _check("razer_quantize_weights", st)
    return codes, scales, ts


def razer_quantize_weights_batch(Ws, fmt="weight", *, codes=None, scales=None, ts=None, stream=None):
    """Quantize several weight matrices (same dtype and device) in one call.
    Returns (list of codes, list of scales, ts [count] f32); matrix i's
    results equal razer_quantize_weights(Ws[i])."""
    n = len(Ws)
    dev = Ws[0].device if n else torch.device("cuda")
    dt = _DT.get(Ws[0].dtype, -1) if n else 0
    codes = [torch.empty((w.shape[0], w.shape[1] // 2), dtype=torch.uint8, device=dev) for w in Ws] if codes is None else codes
    scales = [torch.empty((w.shape[0], w.shape[1] // 16), dtype=torch.uint8, device=dev) for w in Ws] if scales is None else scales
    ts = torch.empty(max(n, 1), dtype=torch.float32, device=dev) if ts is None else ts
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    arr = lambda ts_: (vp * max(n, 1))(*[t.data_ptr() for t in ts_])
    Ns = (i64 * max(n, 1))(*[w.shape[0] for w in Ws])
    Ks = (i64 * max(n, 1))(*[w.shape[1] for w in Ws])
    st = load().razer_quantize_weights_batch(n, arr(Ws), dt, Ns, Ks, arr(codes), arr(scales), _p(ts), _fmt(fmt),
                                             _stream(stream))
    _check("razer_quantize_weights_batch", st)
    return codes, scales, ts[:n]


def razer_quantize_acts(X: torch.Tensor, ts_in: torch.Tensor | None = None, fmt="act", *, hist: bool = True,
                        codes=None, scales=None, ts_out=None, meta_hist=None, stream=None):
    """Quantize activations X [M, K]. ts_in (device f32 [1]) = static scale,
    None = dynamic. Returns (codes, scales, ts_out, meta_hist [4] i64 or None)."""
    M, K = X.shape
    dev = X.device
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev) if codes is None else codes
    scales = torch.empty((M, K // 16), dtype=torch.uint8, device=dev) if scales is None else scales
    ts_out = torch.empty(1, dtype=torch.float32, device=dev) if ts_out is None else ts_out
    if hist and meta_hist is None:
        meta_hist = torch.empty(4, dtype=torch.int64, device=dev)
    st = load().razer_quantize_acts(_p(X), _DT.get(X.dtype, -1), M, K, _p(ts_in), _p(codes), _p(scales), _p(ts_out),
                                    _p(meta_hist) if hist else None, _fmt(fmt), _stream(stream))
    _check("razer_quantize_acts", st)
    return codes, scales, ts_out, (meta_hist if hist else None)


def razer_dequant(codes: torch.Tensor, scales: torch.Tensor, ts: torch.Tensor, fmt="weight",
                  out_dtype=torch.float32, *, out=None, stream=None):
    R, K2 = codes.shape
    K = 2 * K2
    out = torch.empty((R, K), dtype=out_dtype, device=codes.device) if out is None else out
    st = load().razer_dequant(_p(codes), _p(scales), _p(ts), _fmt(fmt), R, K, _p(out), _DT.get(out.dtype, -1), _stream(stream))
    _check("razer_dequant", st)
    return out


def razer_workspace_size(op: int, m_or_b: int, N: int, K: int) -> int:
    return int(load().razer_workspace_size(op, m_or_b, N, K))


def _workspace(op, m, N, K, dev, workspace):
    need = razer_workspace_size(op, m, N, K)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    return workspace, (workspace.numel() * workspace.element_size() if workspace is not None else 0)


def razer_gemv(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, ts: torch.Tensor, fmt="weight",
               out_dtype=torch.float32, *, out=None, workspace=None, stream=None):
    """y [B, N] = ts * x [B, K] . deq(W [N, K])^T with 1 <= B <= 32."""
    B, K = x.shape
    N = codes.shape[0]
    out = torch.empty((B, N), dtype=out_dtype, device=x.device) if out is None else out
    workspace, wsb = _workspace(RAZER_OP_GEMV, B, N, K, x.device, workspace)
    st = load().razer_gemv(_p(x), _DT.get(x.dtype, -1), B, _p(codes), _p(scales), _p(ts), _fmt(fmt), N, K, _p(out),
                           _DT.get(out.dtype, -1), _p(workspace), wsb, _stream(stream))
    _check("razer_gemv", st)
    return out


def razer_gemm_w4a4(codes_a: torch.Tensor, scales_a: torch.Tensor, ts_a: torch.Tensor, codes_w: torch.Tensor,
                    scales_w: torch.Tensor, ts_w: torch.Tensor, afmt="act", wfmt="weight", out_dtype=torch.bfloat16, *,
                    out=None, workspace=None, stream=None):
    """Y [M, N] = ts_a * ts_w * deq(A [M, K]) . deq(W [N, K])^T, both operands RaZeR-packed."""
    M, N, K = codes_a.shape[0], codes_w.shape[0], codes_w.shape[1] * 2
    dev = codes_w.device
    out = torch.empty((M, N), dtype=out_dtype, device=dev) if out is None else out
    workspace, wsb = _workspace(RAZER_OP_GEMM_W4A4, M, N, K, dev, workspace)
    st = load().razer_gemm_w4a4(_p(codes_a), _p(scales_a), _p(ts_a), _fmt(afmt), M, _p(codes_w), _p(scales_w), _p(ts_w),
                                _fmt(wfmt), N, K, _p(out), _DT.get(out.dtype, -1), _p(workspace), wsb, _stream(stream))
    _check("razer_gemm_w4a4", st)
    return out


def razer_gemm_w4a4_online(X: torch.Tensor, codes_w: torch.Tensor, scales_w: torch.Tensor, ts_w: torch.Tensor,
                           ts_in: torch.Tensor | None = None, afmt="act", wfmt="weight", out_dtype=torch.bfloat16, *,
                           keep_codes: bool = False, hist: bool = False, out=None, workspace=None, stream=None):
    """Quantize activations X [M, K] and multiply with the packed weights W [N, K]
    in one call. Returns (Y [M, N], ts_a [1], (codes_a, scales_a) or None, meta_hist or None)."""
    M, K = X.shape
    N = codes_w.shape[0]
    dev = X.device
    out = torch.empty((M, N), dtype=out_dtype, device=dev) if out is None else out
    ts_a = torch.empty(1, dtype=torch.float32, device=dev)
    ca = torch.empty((M, K // 2), dtype=torch.uint8, device=dev) if keep_codes else None
    sa = torch.empty((M, K // 16), dtype=torch.uint8, device=dev) if keep_codes else None
    mh = torch.empty(4, dtype=torch.int64, device=dev) if hist else None
    workspace, wsb = _workspace(RAZER_OP_GEMM_W4A4, M, N, K, dev, workspace)
    st = load().razer_gemm_w4a4_online(_p(X), _DT.get(X.dtype, -1), M, _p(ts_in), _fmt(afmt), _p(ca), _p(sa), _p(ts_a), _p(mh),
                                       _p(codes_w), _p(scales_w), _p(ts_w), _fmt(wfmt), N, K, _p(out), _DT.get(out.dtype, -1),
                                       _p(workspace), wsb, _stream(stream))
    _check("razer_gemm_w4a4_online", st)
    return out, ts_a, ((ca, sa) if keep_codes else None), mh


def _varr(V):
    return (ctypes.c_float * max(len(V), 1))(*[float(v) for v in V])


def razer_quantize_variant(X: torch.Tensor, block: int, scale_fmt, V, *, stream=None):
    """RaZeR quantization with a `block`-element block and special values V.
    Returns (codes [R, K/2], scales [R, K/block], ts [1])."""
    R, K = X.shape
    dev = X.device
    codes = torch.empty((R, K // 2), dtype=torch.uint8, device=dev)
    wide = _fmt(scale_fmt) == RAZER_SCALE_F16
    scales = torch.empty((R, (K // block) * (2 if wide else 1)), dtype=torch.uint8, device=dev)
    ts = torch.empty(1, dtype=torch.float32, device=dev)
    st = load().razer_quantize_variant(_p(X), _DT.get(X.dtype, -1), R, K, block, _fmt(scale_fmt), _varr(V), len(V), _p(codes),
                                       _p(scales), _p(ts), _stream(stream))
    _check("razer_quantize_variant", st)
    return codes, scales, ts


def razer_dequant_variant(codes: torch.Tensor, scales: torch.Tensor, ts: torch.Tensor, block: int, scale_fmt, V,
                          out_dtype=torch.float32, *, out=None, stream=None):
    """Decode a razer_quantize_variant tensor to [R, K]: (q*s)*ts rounded once to out_dtype."""
    R, K2 = codes.shape
    K = 2 * K2
    out = torch.empty((R, K), dtype=out_dtype, device=codes.device) if out is None else out
    st = load().razer_dequant_variant(_p(codes), _p(scales), _p(ts), R, K, block, _fmt(scale_fmt), _varr(V), len(V), _p(out),
                                      _DT.get(out.dtype, -1), _stream(stream))
    _check("razer_dequant_variant", st)
    return out


def razer_gemv_variant(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, ts: torch.Tensor, block: int, scale_fmt, V,
                       out_dtype=torch.float32, *, out=None, workspace=None, stream=None):
    """y [B, N] = ts * x [B, K] . deq(W [N, K])^T for a razer_quantize_variant weight tensor, 1 <= B <= 32."""
    B, K = x.shape
    N = codes.shape[0]
    out = torch.empty((B, N), dtype=out_dtype, device=x.device) if out is None else out
    workspace, wsb = _workspace(RAZER_OP_GEMV, B, N, K, x.device, workspace)
    st = load().razer_gemv_variant(_p(x), _DT.get(x.dtype, -1), B, _p(codes), _p(scales), _p(ts), block, _fmt(scale_fmt),
                                   _varr(V), len(V), N, K, _p(out), _DT.get(out.dtype, -1), _p(workspace), wsb, _stream(stream))
    _check("razer_gemv_variant", st)
    return out


def razer_gemm_variant(X: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, ts: torch.Tensor, block: int, scale_fmt, V,
                       out_dtype=torch.bfloat16, *, out=None, workspace=None, stream=None):
    """Y [M, N] = ts * X [M, K] . deq(W [N, K])^T for a razer_quantize_variant weight tensor (tcgen05 GEMM)."""
    M, K = X.shape
    N = codes.shape[0]
    out = torch.empty((M, N), dtype=out_dtype, device=X.device) if out is None else out
    workspace, wsb = _workspace(RAZER_OP_GEMM_VARIANT, M, N, K, X.device, workspace)
    st = load().razer_gemm_variant(_p(X), _DT.get(X.dtype, -1), M, _p(codes), _p(scales), _p(ts), block, _fmt(scale_fmt),
                                   _varr(V), len(V), N, K, _p(out), _DT.get(out.dtype, -1), _p(workspace), wsb, _stream(stream))
    _check("razer_gemm_variant", st)
    return out


def razer_quant_error_variant(X: torch.Tensor, block: int, scale_fmt, V, codes, scales, ts, *, out=None, stream=None):
    """sum (X - deq(X))^2 (double, device [1]) for a tensor of razer_quantize_variant."""
    R, K = X.shape
    out = torch.empty(1, dtype=torch.float64, device=X.device) if out is None else out
    st = load().razer_quant_error_variant(_p(X), _DT.get(X.dtype, -1), R, K, block, _fmt(scale_fmt), _varr(V), len(V), _p(codes),
                                          _p(scales), _p(ts), _p(out), _stream(stream))
    _check("razer_quant_error_variant", st)
    return out


def razer_quant_error(X: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, ts: torch.Tensor, fmt="weight", *,
                      out=None, stream=None) -> torch.Tensor:
    """sum (X - deq(X))^2 over the tensor in double (device [1] f64)."""
    R, K = X.shape
    out = torch.empty(1, dtype=torch.float64, device=X.device) if out is None else out
    st = load().razer_quant_error(_p(X), _DT.get(X.dtype, -1), R, K, _p(codes), _p(scales), _p(ts), _fmt(fmt), _p(out),
                                  _stream(stream))
    _check("razer_quant_error", st)
    return out


def razer_gemv_batch(problems, fmt="weight", out_dtype=torch.float32, *, outs=None, workspace=None, stream=None):
    """Several independent GEMVs in one call: problems = [(x, codes, scales,
    ts), ...] (same activation dtype and device). Returns [y_i [B_i, N_i]]."""
    n = len(problems)
    if n == 0:
        return []
    dev = problems[0][0].device
    outs = [torch.empty((x.shape[0], c.shape[0]), dtype=out_dtype, device=dev) for x, c, _, _ in problems] if outs is None else outs
    arr = (GemvProblem * n)(*[GemvProblem(x.data_ptr(), x.shape[0], c.data_ptr(), s.data_ptr(), t.data_ptr(), c.shape[0], x.shape[1],
                                          y.data_ptr()) for (x, c, s, t), y in zip(problems, outs)])
    L = load()
    need = int(L.razer_gemv_batch_workspace_size(n, arr))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.razer_gemv_batch(n, arr, _DT.get(problems[0][0].dtype, -1), _fmt(fmt), _DT.get(out_dtype, -1), _p(workspace), wsb,
                            _stream(stream))
    _check("razer_gemv_batch", st)
    return outs


def razer_gemv_batch_workspace_size(problems) -> int:
    """Workspace bytes razer_gemv_batch needs for problems [(x, codes, scales, ts), ...]."""
    n = len(problems)
    arr = (GemvProblem * max(n, 1))(*[GemvProblem(x.data_ptr(), x.shape[0], c.data_ptr(), s.data_ptr(), t.data_ptr(), c.shape[0],
                                                  x.shape[1], 0) for x, c, s, t in problems])
    return int(load().razer_gemv_batch_workspace_size(n, arr))


def razer_gemv_noalloc(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, ts: torch.Tensor, fmt="weight",
                       out_dtype=torch.float32, *, out=None, stream=None):
    """razer_gemv without a workspace: the split-K scratch is a fixed array
    inside the library (for callers that cannot allocate device memory)."""
    B, K = x.shape
    N = codes.shape[0]
    out = torch.empty((B, N), dtype=out_dtype, device=x.device) if out is None else out
    st = load().razer_gemv_noalloc(_p(x), _DT.get(x.dtype, -1), B, _p(codes), _p(scales), _p(ts), _fmt(fmt), N, K,
                                   _p(out), _DT.get(out.dtype, -1), _stream(stream))
    _check("razer_gemv_noalloc", st)
    return out


def razer_gemv_noalloc_max_scratch() -> int:
    return int(load().razer_gemv_noalloc_max_scratch())


def razer_gemm(X: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, ts: torch.Tensor, fmt="weight",
               out_dtype=torch.bfloat16, *, out=None, workspace=None, stream=None):
    """Y [M, N] = ts * X [M, K] . deq(W [N, K])^T on the tcgen05 tensor cores."""
    M, K = X.shape
    N = codes.shape[0]
    out = torch.empty((M, N), dtype=out_dtype, device=X.device) if out is None else out
    workspace, wsb = _workspace(RAZER_OP_GEMM, M, N, K, X.device, workspace)
    st = load().razer_gemm(_p(X), _DT.get(X.dtype, -1), M, _p(codes), _p(scales), _p(ts), _fmt(fmt), N, K, _p(out),
                           _DT.get(out.dtype, -1), _p(workspace), wsb, _stream(stream))
    _check("razer_gemm", st)
    return out


def razer_get_device_status(stream=None) -> int:
    """Synchronises the stream; returns and clears the device error word."""
    return int(load().razer_get_device_status(_stream(stream)))


def razer_status_string(status: int) -> str:
    return load().razer_status_string(status).decode()


def razer_version() -> int:
    return int(load().razer_version())


RAZER_QPATH_TWO_PASS, RAZER_QPATH_SINGLE_PASS = 0, 1
QUANTIZE_PATHS = {"two_pass": RAZER_QPATH_TWO_PASS, "single_pass": RAZER_QPATH_SINGLE_PASS}


def razer_set_quantize_path(path: str) -> str:
    """Selects the dynamic-scale quantizer path ("two_pass", the default, or
    "single_pass"); returns the previous one."""
    if path not in QUANTIZE_PATHS:
        raise ValueError(f"unknown quantizer path {path!r}")
    prev = int(load().razer_set_quantize_path(QUANTIZE_PATHS[path]))
    return "single_pass" if prev == RAZER_QPATH_SINGLE_PASS else "two_pass"


def razer_debug_set_fault_injection(on: bool) -> bool:
    """Test-only: turns the GEMV / GEMM / single-pass quantizer stall
    injection on or off; returns the previous setting."""
    return bool(load().razer_debug_set_fault_injection(1 if on else 0))
