"""RaZeR CPU oracle -- TEST INFRASTRUCTURE ONLY.

Thin ctypes wrapper over ``razer_oracle.c``, a plain single-threaded C
implementation of the RaZeR block quantizer, its decoder and a double-precision
reference product.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the CUDA library
never does, and the two share no code.

Every function follows the RaZeR pages ("RaZeR: Pushing the Limits of NVFP4
Quantization with Redundant Zero Remapping", papernotes.org notes, 关键设计
1-3 and the worked example 一个完整示例; gist.science technical summary,
sections 1 and 2.1-2.2); the readings taken where the pages are open are
listed in the header of ``razer_oracle.c``.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(hand-worked vectors from the worked example, library conversions, brute-force
enumeration with exact rationals, invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "razer_oracle.c")
_LIB_PATH = os.path.join(_HERE, "librazer_oracle.so")

FMT_WEIGHT = 0  # E3M3 scale + 2-bit meta, V_w = {+5, -5, +8, -8}
FMT_ACT = 1  # E4M3 scale + 1-bit meta, V_a = {+5, -5}
FMT_NVFP4 = 2  # E4M3 scale, no remap
SCALE_F16 = 4  # format variants only: FP16 block scale, meta in bits 15..14, no tensor scale
FORMATS = {"weight": FMT_WEIGHT, "act": FMT_ACT, "nvfp4": FMT_NVFP4}

F16, BF16, F32 = 0, 1, 2

BUILD_CMD = [
    "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
    "-fPIC", "-shared", "-o", _LIB_PATH, _SRC, "-lm",
]


def build(force: bool = False) -> str:
    """Compile the oracle shared object (gcc, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(BUILD_CMD)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        vp, i64, f32, f64, u8p = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p
        L.ro_f16_to_double.argtypes = [ctypes.c_uint16]
        L.ro_f16_to_double.restype = f64
        L.ro_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.ro_bf16_to_double.restype = f64
        L.ro_float_to_f16.argtypes = [f32]
        L.ro_float_to_f16.restype = ctypes.c_uint16
        L.ro_float_to_bf16.argtypes = [f32]
        L.ro_float_to_bf16.restype = ctypes.c_uint16
        L.ro_scale_value.argtypes = [ctypes.c_int, ctypes.c_int]
        L.ro_scale_value.restype = f64
        L.ro_scale_max.argtypes = [ctypes.c_int]
        L.ro_scale_max.restype = f64
        L.ro_scale_encode.argtypes = [ctypes.c_int, f32]
        L.ro_scale_encode.restype = ctypes.c_int
        L.ro_num_specials.argtypes = [ctypes.c_int]
        L.ro_num_specials.restype = ctypes.c_int
        L.ro_special_value.argtypes = [ctypes.c_int, ctypes.c_int]
        L.ro_special_value.restype = f64
        L.ro_fp4_value.argtypes = [ctypes.c_int, ctypes.c_int, f64]
        L.ro_fp4_value.restype = f64
        L.ro_tensor_scale.argtypes = [vp, ctypes.c_int, i64, ctypes.c_int]
        L.ro_tensor_scale.restype = f32
        L.ro_quantize_block.argtypes = [vp, f32, ctypes.c_int, u8p, u8p, vp, vp]
        L.ro_quantize_block.restype = None
        L.ro_quantize.argtypes = [vp, ctypes.c_int, i64, i64, ctypes.c_int, f32, u8p, u8p, vp]
        L.ro_quantize.restype = ctypes.c_int
        L.ro_dequant.argtypes = [u8p, u8p, f32, ctypes.c_int, i64, i64, ctypes.c_int, vp]
        L.ro_dequant.restype = ctypes.c_int
        L.ro_gemm_ref.argtypes = [vp, ctypes.c_int, i64, u8p, u8p, f32, ctypes.c_int, i64, i64, vp, i64, vp]
        L.ro_quantize_46.argtypes = [vp, ctypes.c_int, i64, i64, f32, u8p, u8p, vp]
        L.ro_quant_sse.argtypes = [vp, ctypes.c_int, i64, i64, u8p, u8p, f32, ctypes.c_int]
        L.ro_quant_sse.restype = f64
        L.ro_quantize_generic.argtypes = [vp, ctypes.c_int, i64, i64, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, f32, u8p, u8p]
        L.ro_quant_sse_generic.argtypes = [vp, ctypes.c_int, i64, i64, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, u8p, u8p, f32]
        L.ro_quant_sse_generic.restype = f64
        L.ro_dequant_generic.argtypes = [u8p, u8p, f32, i64, i64, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, ctypes.c_int, vp]
        L.ro_dequant_generic.restype = ctypes.c_int
        L.ro_gemv_generic.argtypes = [vp, ctypes.c_int, i64, u8p, u8p, f32, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, i64, i64, vp]
        L.ro_gemv_generic.restype = ctypes.c_int
        L.ro_gemm_w4a4_ref.argtypes = [u8p, u8p, f32, ctypes.c_int, i64, u8p, u8p, f32, ctypes.c_int, i64, i64, vp, i64, vp]
        L.ro_gemm_ref.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_bits(x) -> tuple[np.ndarray, int]:
    """Accept a numpy float16/float32 array, or a uint16 array tagged by the
    caller as bfloat16 via ``bf16_bits``; returns (contiguous array, dtype id)."""
    if isinstance(x, Bf16Bits):
        return np.ascontiguousarray(x.bits, dtype=np.uint16), BF16
    x = np.asarray(x)
    if x.dtype == np.float16:
        return np.ascontiguousarray(x), F16
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), F32
    raise TypeError(f"oracle input must be float16, float32 or Bf16Bits, got {x.dtype}")


class Bf16Bits:
    """Raw bfloat16 payload (numpy has no bfloat16): ``bits`` is uint16."""

    def __init__(self, bits: np.ndarray):
        self.bits = np.asarray(bits, dtype=np.uint16)
        self.shape = self.bits.shape


def f16_to_double(h: int) -> float:
    return lib().ro_f16_to_double(h)


def bf16_to_double(b: int) -> float:
    return lib().ro_bf16_to_double(b)


def float_to_f16_bits(f: float) -> int:
    return lib().ro_float_to_f16(f)


def float_to_bf16_bits(f: float) -> int:
    return lib().ro_float_to_bf16(f)


def scale_value(fmt: int, code: int) -> float:
    return lib().ro_scale_value(fmt, code)


def scale_max(fmt: int) -> float:
    return lib().ro_scale_max(fmt)


def scale_encode(fmt: int, s_f: float) -> int:
    return lib().ro_scale_encode(fmt, s_f)


def num_specials(fmt: int) -> int:
    return lib().ro_num_specials(fmt)


def special_value(fmt: int, meta: int) -> float:
    return lib().ro_special_value(fmt, meta)


def fp4_value(code: int, v: float | None) -> float:
    return lib().ro_fp4_value(code, 0 if v is None else 1, 0.0 if v is None else v)


def tensor_scale(x, fmt: int) -> float:
    a, dt = _as_bits(x)
    return float(lib().ro_tensor_scale(_ptr(a), dt, a.size, fmt))


def quantize_block(x16, ts: float, fmt: int):
    """One 16-element block (binary32 values). Returns
    (codes[16] uint8, scale_byte, xs[16] float32, sse_delta[4] float64)."""
    x = np.ascontiguousarray(np.asarray(x16, dtype=np.float32).reshape(16))
    codes = np.zeros(16, np.uint8)
    sb = np.zeros(1, np.uint8)
    xs = np.zeros(16, np.float32)
    dl = np.zeros(4, np.float64)
    lib().ro_quantize_block(_ptr(x), ts, fmt, _ptr(codes), _ptr(sb), _ptr(xs), _ptr(dl))
    return codes, int(sb[0]), xs, dl


def quantize(x, fmt: int, ts: float | None = None):
    """Quantize a [R, K] tensor. Returns (codes [R, K/2] u8, scales [R, K/16] u8,
    ts, hist[8] u64).  ts=None computes the tensor scale from x."""
    a, dt = _as_bits(x)
    R, K = a.shape
    if ts is None:
        ts = tensor_scale(x, fmt)
    codes = np.zeros((R, K // 2), np.uint8)
    scales = np.zeros((R, K // 16), np.uint8)
    hist = np.zeros(8, np.uint64)
    rc = lib().ro_quantize(_ptr(a), dt, R, K, fmt, ts, _ptr(codes), _ptr(scales), _ptr(hist))
    if rc != 0:
        raise ValueError("oracle quantize: K must be a multiple of 16")
    return codes, scales, float(np.float32(ts)), hist


def dequant(codes: np.ndarray, scales: np.ndarray, ts: float, fmt: int, out_dtype: str = "f32"):
    """Decode to [R, K]: f32 values, or uint16 bit patterns for 'f16'/'bf16'."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    R, K2 = codes.shape
    K = K2 * 2
    odt = {"f16": F16, "bf16": BF16, "f32": F32}[out_dtype]
    out = np.zeros((R, K), np.float32 if odt == F32 else np.uint16)
    rc = lib().ro_dequant(_ptr(codes), _ptr(scales), ts, fmt, R, K, odt, _ptr(out))
    if rc != 0:
        raise ValueError("oracle dequant failed")
    return out


def gemm_ref(x, codes: np.ndarray, scales: np.ndarray, ts: float, fmt: int, rows=None) -> np.ndarray:
    """r[m, n] = ts * sum_k x[m, k] * (q*s)[n, k] in double. x is [M, K]."""
    a, dt = _as_bits(x)
    M, K = a.shape
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    N = codes.shape[0]
    if rows is None:
        out = np.zeros((M, N), np.float64)
        rc = lib().ro_gemm_ref(_ptr(a), dt, M, _ptr(codes), _ptr(scales), ts, fmt, N, K, None, 0, _ptr(out))
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        out = np.zeros((r.size, N), np.float64)
        rc = lib().ro_gemm_ref(_ptr(a), dt, M, _ptr(codes), _ptr(scales), ts, fmt, N, K, _ptr(r), r.size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle gemm_ref failed")
    return out


def gemm_w4a4_ref(codes_a: np.ndarray, scales_a: np.ndarray, ts_a: float, afmt: int, codes_w: np.ndarray,
                  scales_w: np.ndarray, ts_w: float, wfmt: int, rows=None) -> np.ndarray:
    """r[m, n] = ts_a * ts_w * sum_k (q*s)_a[m, k] (q*s)_w[n, k] in double:
    both operands RaZeR-packed ([M, K/2] / [M, K/16] and [N, K/2] / [N, K/16])."""
    ca = np.ascontiguousarray(codes_a, dtype=np.uint8)
    sa = np.ascontiguousarray(scales_a, dtype=np.uint8)
    cw = np.ascontiguousarray(codes_w, dtype=np.uint8)
    sw = np.ascontiguousarray(scales_w, dtype=np.uint8)
    M, K = ca.shape[0], ca.shape[1] * 2
    N = cw.shape[0]
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((M if r is None else r.size, N), np.float64)
    rc = lib().ro_gemm_w4a4_ref(_ptr(ca), _ptr(sa), ts_a, afmt, M, _ptr(cw), _ptr(sw), ts_w, wfmt, N, K,
                                None if r is None else _ptr(r), 0 if r is None else r.size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle gemm_w4a4_ref failed")
    return out


def quantize_46(x, ts: float | None = None):
    """FourOverSix quantization (plain NVFP4 encoding, per-block choice of
    the amax -> 6 or amax -> 4 scale). ts None = amax / (6 * 448).
    Returns (codes, scales, ts, blocks that took 4)."""
    a, dt = _as_bits(x)
    R, K = a.shape
    if ts is None:
        ts = tensor_scale(x, FMT_NVFP4)
    codes = np.zeros((R, K // 2), np.uint8)
    scales = np.zeros((R, K // 16), np.uint8)
    n4 = np.zeros(1, np.uint64)
    rc = lib().ro_quantize_46(_ptr(a), dt, R, K, ts, _ptr(codes), _ptr(scales), _ptr(n4))
    if rc != 0:
        raise ValueError("oracle quantize_46: K must be a multiple of 16")
    return codes, scales, float(np.float32(ts)), int(n4[0])


def quant_sse(x, codes: np.ndarray, scales: np.ndarray, ts: float, fmt: int) -> float:
    """sum (x - q*s*ts)^2 over the tensor, in double, row-major order."""
    a, dt = _as_bits(x)
    R, K = a.shape
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    return float(lib().ro_quant_sse(_ptr(a), dt, R, K, _ptr(codes), _ptr(scales), ts, fmt))


def quantize_generic(x, block: int, sfmt: int, V, ts: float | None = None):
    """RaZeR quantization with a block of `block` elements and special values
    V (scale format sfmt: 0 = E3M3 + 2 meta bits, 1/2 = E4M3 + 1 meta bit,
    SCALE_F16 = FP16 scale words with the meta in bits 15..14 and no tensor
    scale). ts None = amax / (6 * S_max(sfmt)) (1 for SCALE_F16). Returns
    (codes, scales [R, K/block] bytes or [R, 2 K/block] for 16-bit words, ts)."""
    a, dt = _as_bits(x)
    R, K = a.shape
    if ts is None:
        ts = 1.0 if sfmt == SCALE_F16 else tensor_scale(x, sfmt)
    v = np.ascontiguousarray(np.asarray(V, dtype=np.float64).reshape(-1))
    codes = np.zeros((R, K // 2), np.uint8)
    scales = np.zeros((R, (K // block) * (2 if sfmt == SCALE_F16 else 1)), np.uint8)
    rc = lib().ro_quantize_generic(_ptr(a), dt, R, K, block, sfmt, _ptr(v) if v.size else None, v.size, ts, _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError("oracle quantize_generic: bad block size")
    return codes, scales, float(np.float32(ts))


def dequant_generic(codes: np.ndarray, scales: np.ndarray, ts: float, block: int, sfmt: int, V, out_dtype: str = "f32"):
    """Decode a variant tensor (codes [R, K/2], scales as quantize_generic
    returns them) to [R, K]: f32 values, or uint16 bit patterns for 'f16'/'bf16'."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    R, K2 = codes.shape
    K = K2 * 2
    v = np.ascontiguousarray(np.asarray(V, dtype=np.float64).reshape(-1))
    odt = {"f16": F16, "bf16": BF16, "f32": F32}[out_dtype]
    out = np.zeros((R, K), np.float32 if odt == F32 else np.uint16)
    rc = lib().ro_dequant_generic(_ptr(codes), _ptr(scales), ts, R, K, block, sfmt, _ptr(v) if v.size else None, v.size, odt,
                                  _ptr(out))
    if rc != 0:
        raise ValueError("oracle dequant_generic: bad block size")
    return out


def gemv_generic(x, codes: np.ndarray, scales: np.ndarray, ts: float, block: int, sfmt: int, V) -> np.ndarray:
    """r[b, n] = ts * sum_k x[b, k] * (q*s)[n, k] in double for a variant
    weight tensor; x is [B, K] (fp16/bf16 torch tensor or numpy)."""
    a, dt = _as_bits(x)
    B, K = a.shape
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    N = codes.shape[0]
    v = np.ascontiguousarray(np.asarray(V, dtype=np.float64).reshape(-1))
    out = np.zeros((B, N), np.float64)
    rc = lib().ro_gemv_generic(_ptr(a), dt, B, _ptr(codes), _ptr(scales), ts, block, sfmt, _ptr(v) if v.size else None, v.size,
                               N, K, _ptr(out))
    if rc != 0:
        raise ValueError("oracle gemv_generic failed")
    return out


def quant_sse_generic(x, block: int, sfmt: int, V, codes: np.ndarray, scales: np.ndarray, ts: float) -> float:
    a, dt = _as_bits(x)
    R, K = a.shape
    v = np.ascontiguousarray(np.asarray(V, dtype=np.float64).reshape(-1))
    return float(lib().ro_quant_sse_generic(_ptr(a), dt, R, K, block, sfmt, _ptr(v) if v.size else None, v.size,
                                            _ptr(np.ascontiguousarray(codes)), _ptr(np.ascontiguousarray(scales)), ts))

