"""Host-side checks of the C ABI: the library loads, exports every function
include/razer.h declares, and rejects bad arguments before launching anything
(no compute calls: these run without a GPU)."""
import ctypes
import os
import re

import pytest

from bit_quantization_razer_b200 import razer
from bit_quantization_razer_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return razer.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "razer.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(razer_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "razer_gemv" in names and "razer_quantize_weights" in names
    for n in names:
        assert hasattr(lib, n), n
    for n in razer.EXPORTED:
        assert n in names


def test_plain_c_consumer(lib, tmp_path):
    # the header compiles as C99 with every warning an error, and a C program
    # linked against the library gets the documented statuses
    import subprocess

    libdir = os.path.join(ROOT, "bit_quantization_razer_b200")
    exe = str(tmp_path / "abi_consumer")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "abi_consumer.c"), "-L", libdir, "-lrazer", "-Wl,-rpath," + libdir,
                    "-o", exe], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert "all checks passed" in out.stdout


def test_status_strings(lib):
    for s in range(9):
        assert razer.razer_status_string(s)
    assert razer.razer_status_string(3) == "misaligned pointer"
    assert razer.razer_version() >= 100


FAKE = ctypes.c_void_p(0x1000)  # 16-byte aligned; never dereferenced (validation fails first)
ODD = ctypes.c_void_p(0x1001)


def test_quantize_validation(lib):
    q = lib.razer_quantize_weights
    assert q(None, 0, 4, 32, FAKE, FAKE, FAKE, 0, None) == 1
    assert q(FAKE, 0, 4, 32, FAKE, FAKE, FAKE, 1, None) == 6       # ACT format is for activations
    assert q(FAKE, 0, 4, 32, FAKE, FAKE, FAKE, 7, None) == 1       # unknown format
    assert q(FAKE, 2, 4, 32, FAKE, FAKE, FAKE, 0, None) == 4       # fp32 input not supported
    assert q(FAKE, 0, 4, 24, FAKE, FAKE, FAKE, 0, None) == 2       # K % 16
    assert q(FAKE, 0, -1, 32, FAKE, FAKE, FAKE, 0, None) == 2
    assert q(ODD, 0, 4, 32, FAKE, FAKE, FAKE, 0, None) == 3
    assert q(FAKE, 0, 4, 32, ODD, FAKE, FAKE, 0, None) == 3
    b = lib.razer_quantize_weights_batch
    arr = lambda *v: (ctypes.c_void_p * len(v))(*v)
    i64s = lambda *v: (ctypes.c_int64 * len(v))(*v)
    assert b(0, None, 0, None, None, None, None, None, 0, None) == 0                     # empty batch
    assert b(-1, None, 0, None, None, None, None, None, 0, None) == 1
    assert b(2, arr(FAKE, FAKE), 0, i64s(4, 4), i64s(32, 32), arr(FAKE, FAKE), arr(FAKE, FAKE), None, 0, None) == 1
    assert b(2, arr(FAKE, FAKE), 0, i64s(4, 4), i64s(32, 24), arr(FAKE, FAKE), arr(FAKE, FAKE), FAKE, 0, None) == 2
    assert b(2, arr(FAKE, ODD), 0, i64s(4, 4), i64s(32, 32), arr(FAKE, FAKE), arr(FAKE, FAKE), FAKE, 0, None) == 3
    assert b(2, arr(FAKE, FAKE), 0, i64s(4, 4), i64s(32, 32), arr(FAKE, FAKE), arr(FAKE, FAKE), FAKE, 1, None) == 6
    assert b(1, arr(FAKE), 2, i64s(4), i64s(32), arr(FAKE), arr(FAKE), FAKE, 0, None) == 4
    a = lib.razer_quantize_acts
    assert a(FAKE, 1, 4, 32, None, FAKE, FAKE, None, None, 1, None) == 1
    assert a(FAKE, 1, 4, 32, None, FAKE, FAKE, FAKE, None, 0, None) == 6
    assert a(FAKE, 1, 4, 32, ODD, FAKE, FAKE, FAKE, None, 1, None) == 3


def test_gemv_gemm_validation(lib):
    g = lib.razer_gemv
    args = lambda B, N, K, ws=None, wsb=0: (FAKE, 0, B, FAKE, FAKE, FAKE, 0, N, K, FAKE, 2, ws, wsb, None)
    assert g(*args(0, 64, 128)) == 2
    assert g(*args(33, 64, 128)) == 2
    assert g(*args(1, 64, 24)) == 2          # K % 16 (the only K-shape error)
    assert g(*args(33, 64, 96)) == 2         # B, with a K outside the 128-k chunking
    assert g(*args(1, 64, 128)) == 5         # workspace missing
    assert g(FAKE, 2, 1, FAKE, FAKE, FAKE, 0, 64, 128, FAKE, 2, None, 0, None) == 4
    m = lib.razer_gemm
    assert m(FAKE, 1, 64, FAKE, FAKE, FAKE, 0, 64, 24, FAKE, 1, None, 0, None) == 2   # K % 16
    # K % 64 != 0 and N % 16 != 0 are served (decode-once path): they need its workspace
    assert m(FAKE, 1, 64, FAKE, FAKE, FAKE, 0, 64, 96, FAKE, 1, None, 0, None) == 5
    assert m(FAKE, 1, 64, FAKE, FAKE, FAKE, 0, 40, 128, FAKE, 1, None, 0, None) == 5
    assert razer.razer_workspace_size(razer.RAZER_OP_GEMM, 64, 40, 96) == 40 * 96 * 2
    assert m(None, 1, 64, FAKE, FAKE, FAKE, 0, 64, 128, FAKE, 1, None, 0, None) == 1
    w = lib.razer_gemm_w4a4
    wargs = lambda M, N, K, afmt=1, wfmt=0, ts=FAKE, y=FAKE: (FAKE, FAKE, ts, afmt, M, FAKE, FAKE, FAKE, wfmt, N, K, y, 1, None, 0,
                                                              None)
    assert w(*wargs(64, 64, 24)) == 2            # K % 16
    assert w(*wargs(64, 64, 96)) == 5            # K % 64 != 0 is served: workspace missing
    assert w(*wargs(64, 40, 128)) == 5           # N % 16 != 0 likewise
    assert w(*wargs(64, 64, 128, afmt=5)) == 1   # unknown format
    assert w(*wargs(64, 64, 128, ts=None)) == 1
    assert w(*wargs(64, 64, 128, y=ODD)) == 3
    assert w(*wargs(64, 64, 128)) == 5           # workspace missing
    assert w(*wargs(0, 64, 128)) == 0            # empty product
    v = lib.razer_quantize_variant
    vals = lambda *xs: (ctypes.c_float * max(len(xs), 1))(*xs)
    vargs = lambda block, sfmt, V, K=128: (FAKE, 0, 4, K, block, sfmt, vals(*V), len(V), FAKE, FAKE, FAKE, None)
    assert v(*vargs(24, 0, [5.0])) == 2                  # block size
    assert v(*vargs(64, 0, [5.0], K=96)) == 2            # K % block
    assert v(*vargs(32, 0, [3.0])) == 1                  # an E2M1 magnitude
    assert v(*vargs(32, 0, [10.0])) == 1                 # above 9.5
    assert v(*vargs(32, 0, [2.7])) == 1                  # not a multiple of 0.5
    assert v(*vargs(32, 1, [5.0, -5.0, 7.0])) == 1       # E4M3 has one meta bit
    assert v(*vargs(32, 0, [2.5, -2.5, 9.5, -9.5], K=128)[:4] + (32, 0, vals(2.5, -2.5, 9.5, -9.5), 4, FAKE, FAKE, None, None)) == 1
    d = lib.razer_dequant
    assert d(FAKE, FAKE, FAKE, 3, 4, 32, FAKE, 2, None) == 1
    assert d(FAKE, FAKE, FAKE, 0, 4, 32, FAKE, 5, None) == 1
    assert d(FAKE, FAKE, FAKE, 0, 4, 32, ODD, 2, None) == 3


def test_variant_decode_validation(lib):
    vals = lambda *xs: (ctypes.c_float * max(len(xs), 1))(*xs)
    g = lib.razer_gemv_variant

    def gargs(block=32, sfmt=0, V=(5.0, -5.0), B=1, N=64, K=128, act=0, codes=FAKE, scales=FAKE):
        return (FAKE, act, B, codes, scales, FAKE, block, sfmt, vals(*V), len(V), N, K, FAKE, 2, None, 0, None)

    assert g(*gargs(block=24)) == 2                                   # block size
    assert g(*gargs(block=32, K=96)) == 2                              # K % block
    assert g(*gargs(block=32, K=64 * 3)) == 2                          # K % 128
    assert g(*gargs(B=33)) == 2
    assert g(*gargs(act=2)) == 4                                       # f32 activations
    assert g(*gargs(block=64, sfmt=4)) == 6                            # FP16 scale words: block 128 only
    assert g(*gargs(V=(5.0, -5.0, 9.5, -9.5), act=1)) == 6             # bf16 operand would round (19 * 15 = 285)
    assert g(*gargs(V=(5.0, -5.0, 8.5, -8.5), act=1)) == 5             # 17 * 15 = 255 fits: allowed (no workspace)
    assert g(*gargs(V=(5.0, -5.0, 9.0, -9.0), act=1)) == 5
    assert g(*gargs(V=(5.0, -5.0, 9.5, -9.5), act=0)) == 5             # fp16 operands are exact
    assert g(*gargs(block=128, sfmt=4, V=(9.5, -9.5), act=1)) == 5     # q alone enters the MMA
    assert g(*gargs(block=128, sfmt=4, scales=ODD)) == 3               # 16-bit scale words
    assert g(*gargs(codes=ctypes.c_void_p(0x1008))) == 3
    assert g(*gargs(N=0)) == 0                                         # empty product
    d = lib.razer_dequant_variant
    dargs = lambda block=32, sfmt=0, R=4, K=128, ts=FAKE, out=FAKE, odt=2: (FAKE, FAKE, ts, R, K, block, sfmt, vals(5.0, -5.0), 2,
                                                                            out, odt, None)
    assert d(*dargs(ts=None)) == 1
    assert d(*dargs(out=ODD)) == 3
    assert d(*dargs(odt=5)) == 1
    assert d(*dargs(block=48)) == 2
    assert d(*dargs(block=64, K=96)) == 2
    assert d(*dargs(R=0)) == 0                                         # empty tensor
    # the prefill GEMM on variant weights: every refusal happens before a launch
    m = lib.razer_gemm_variant
    m.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                  ctypes.c_int, ctypes.POINTER(ctypes.c_float), ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    m.restype = ctypes.c_int

    def margs(block=32, sfmt=0, V=(5.0, -5.0), M=256, N=64, K=128, act=0, codes=FAKE, scales=FAKE, ts=FAKE, ws=None, wsb=0, Y=FAKE):
        return (FAKE, act, M, codes, scales, ts, block, sfmt, vals(*V), len(V), N, K, Y, 2, ws, wsb, None)

    assert m(*margs(ts=None)) == 1
    assert m(*margs(block=24)) == 2                                   # block size
    assert m(*margs(block=64, K=96)) == 2                              # K % block
    assert m(*margs(M=-1)) == 2
    assert m(*margs(act=2)) == 4                                       # f32 activations
    assert m(*margs(V=(5.0, -5.0, 9.5, -9.5), act=1)) == 6             # a bf16 copy would round 9.5 x the scale
    assert m(*margs(block=32, sfmt=4, K=96)) == 6                      # FP16 words: whole 64-element k-steps
    assert m(*margs(block=128, sfmt=4, scales=ODD)) == 3               # 16-bit scale words
    assert m(*margs(codes=ctypes.c_void_p(0x1004))) == 3               # 8-byte aligned codes
    assert m(*margs(Y=ODD)) == 3
    assert m(*margs()) == 5                                            # no workspace
    assert m(*margs(ws=ctypes.c_void_p(0x1000), wsb=16)) == 5          # too small
    assert m(*margs(M=0)) == 0 and m(*margs(N=0)) == 0                 # empty products


def test_quantize_path_selector(lib):
    # host-side setting only: no kernel runs
    lib.razer_set_quantize_path.restype = ctypes.c_int
    lib.razer_set_quantize_path.argtypes = [ctypes.c_int]
    assert lib.razer_set_quantize_path(7) == -1
    assert lib.razer_set_quantize_path(-1) == -1
    prev = lib.razer_set_quantize_path(1)
    assert prev == 0  # two-pass is the default
    assert lib.razer_set_quantize_path(0) == 1
    assert lib.razer_set_quantize_path(0) == 0


def test_workspace_size_host_logic(lib):
    assert razer.razer_workspace_size(razer.RAZER_OP_GEMV, 0, 64, 128) == 0
    def split_k(B, N, K):  # per-warp kernel: ~8 CTAs per SM (148 without a GPU), >= 2 chunks per split
        ctas = ((N + 15) // 16 + 3) // 4
        chunks = K // 128
        S = min(-(-148 * 8 // ctas), chunks // 2 if chunks >= 4 else chunks)
        return max(S, 1) * B * N * 4
    # K % 256 == 0: stream-K plan, one CTA per SM, 128-row tiles; one slot of
    # B x 128 fp32 per (CTA, tile) pair, CTAs + tiles - 1 of them -- or the
    # per-warp kernel's need if larger (it also serves 4-byte aligned scales)
    for B, N, K in [(4, 4096, 4096), (1, 14336, 4096), (16, 4096, 14336), (32, 100, 256)]:
        T = (N + 127) // 128
        G = min(148, T * (K // 128))
        tma = (G + T - 1) * B * 128 * 4
        assert razer.razer_workspace_size(razer.RAZER_OP_GEMV, B, N, K) == max(tma, split_k(B, N, K))
    # other K: split-K partials of the per-warp kernel only
    assert razer.razer_workspace_size(razer.RAZER_OP_GEMV, 4, 4096, 4224) == split_k(4, 4096, 4224)
    # GEMM: the decoded 16-bit weight copy for M >= 1024, plus one fp32 [M, N]
    # slice per parallel K split: as many splits as 16384-long accumulation
    # chains K needs, more when the 256x256 output tiles leave SMs idle (each
    # split keeps at least 8 k-steps of 64); 148 SMs without a GPU
    G = razer.RAZER_OP_GEMM

    def splits(M, N, K):
        tiles = -(-M // 256) * -(-N // 256)
        s = -(-K // 16384)
        if 0 < tiles < 148:
            s = max(s, min(148 // tiles, (K // 64) // 8))
        return max(s, 1)

    def slices(M, N, K):
        s = splits(M, N, K)
        return s * M * N * 4 if s > 1 else 0

    assert splits(1023, 4096, 16384) == 2 and splits(8192, 8192, 8192) == 1 and splits(256, 256, 256) == 1
    assert splits(256, 256, 4096) == 8 and splits(512, 28672, 8192) == 1 and splits(2048, 8192, 28672) == 2
    assert razer.razer_workspace_size(G, 8192, 8192, 8192) == 8192 * 8192 * 2
    assert razer.razer_workspace_size(G, 4096, 14336, 4096) == 14336 * 4096 * 2
    # M >= 256 with at most 2^25 weights also decodes once
    assert razer.razer_workspace_size(G, 256, 256, 256) == 256 * 256 * 2
    assert razer.razer_workspace_size(G, 255, 256, 256) == 0
    assert razer.razer_workspace_size(G, 256, 256, 4096) == 256 * 4096 * 2 + slices(256, 256, 4096)
    assert razer.razer_workspace_size(G, 512, 4096, 8192) == 4096 * 8192 * 2 + slices(512, 4096, 8192)
    for M, N, K in ((1023, 4096, 16384), (512, 8192, 16448), (512, 8192, 8192), (255, 256, 4096), (512, 28672, 8192),
                    (512, 8192, 28672), (512, 4112, 8192)):
        assert razer.razer_workspace_size(G, M, N, K) == slices(M, N, K), (M, N, K)
    assert razer.razer_workspace_size(G, 1024, 4096, 16384) == 4096 * 16384 * 2 + slices(1024, 4096, 16384)
    assert razer.razer_workspace_size(G, 2048, 8192, 28672) == 8192 * 28672 * 2 + 2 * 2048 * 8192 * 4
    # variant GEMM: the decoded copy sized for two 16-bit terms (FP16 scale
    # words), the split slices over 2 K, one float
    GV = razer.RAZER_OP_GEMM_VARIANT
    assert razer.razer_workspace_size(GV, 4096, 4096, 4096) == 4096 * 4096 * 4 + slices(4096, 4096, 8192) + 16
    assert razer.razer_workspace_size(GV, 64, 200, 384) == 200 * 384 * 4 + slices(64, 200, 768) + 16
    assert razer.razer_workspace_size(GV, 0, 200, 384) == 0 and razer.razer_workspace_size(GV, 8, 200, 0) == 0
    # W4A4: both decoded operands, the K-chunk partials, 16 bytes for ts_a * ts_w
    W4 = razer.RAZER_OP_GEMM_W4A4
    assert razer.razer_workspace_size(W4, 100, 64, 128) == 100 * 128 * 2 + 64 * 128 * 2 + 16
    assert razer.razer_workspace_size(W4, 100, 64, 16448) == 100 * 16448 * 2 + 64 * 16448 * 2 + 100 * 64 * 4 + 16
    assert razer.razer_workspace_size(W4, 0, 64, 128) == 0
