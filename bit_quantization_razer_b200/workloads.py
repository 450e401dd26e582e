"""Seeded synthetic inputs for the RaZeR hot path (no quantization arithmetic).

The RaZeR pages evaluate on Llama/Qwen weights and activations, which are not
available here; these generators stand in for them with the shapes and value
distributions of the standard workloads:

* weights: i.i.d. N(0, std^2) (std 0.02 for Llama-3-8B-shaped layers, 0.015
  for Llama-3-70B-shaped ones) with 0.1% of the entries, at seeded positions,
  multiplied by 10 before the cast to fp16;
* activation vectors for GEMV/GEMM: N(0, 1);
* online-quantizer activations: rows N(0, 1) with 8 seeded channels scaled
  x50 to mimic activation outlier channels, cast to bf16.

Everything is generated on the host with ``torch.Generator('cpu')`` so the
same tensors feed the CPU oracle and the GPU path.
"""
from __future__ import annotations

import numpy as np
import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def weight(N: int, K: int, *, std: float = 0.02, seed: int = 0, dtype=torch.float16,
           outlier_frac: float = 0.001, outlier_mult: float = 10.0) -> torch.Tensor:
    """[N, K] weight matrix, N(0, std^2) with a seeded 0.1% of entries x10."""
    g = _gen(seed)
    w = torch.empty(N * K, dtype=torch.float32)
    w.normal_(0.0, std, generator=g)
    n_out = int(round(outlier_frac * N * K))
    if n_out:
        pos = torch.randperm(N * K, generator=g)[:n_out]
        w[pos] *= outlier_mult
    return w.view(N, K).to(dtype)


def vectors(B: int, K: int, *, seed: int = 1, dtype=torch.float16) -> torch.Tensor:
    """[B, K] activations, N(0, 1)."""
    g = _gen(seed)
    x = torch.empty(B, K, dtype=torch.float32)
    x.normal_(0.0, 1.0, generator=g)
    return x.to(dtype)


def outlier_activations(M: int, K: int, *, seed: int = 2, n_channels: int = 8,
                        channel_mult: float = 50.0, dtype=torch.bfloat16) -> torch.Tensor:
    """[M, K] activations: rows N(0, 1), 8 seeded channels scaled x50."""
    g = _gen(seed)
    x = torch.empty(M, K, dtype=torch.float32)
    x.normal_(0.0, 1.0, generator=g)
    ch = torch.randperm(K, generator=g)[:n_channels]
    x[:, ch] *= channel_mult
    return x.to(dtype)


def to_numpy_bits(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit payload of an fp16/bf16 CPU tensor as a uint16 array."""
    assert t.dtype in (torch.float16, torch.bfloat16)
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def random_packed(N: int, K: int, fmt: str, *, seed: int = 3, max_scale_code: int | None = None):
    """Random packed weights [N, K] in a RaZeR format: uniform code bytes and
    uniform scale bytes over every valid magnitude code and meta value (a
    synthetic stand-in that exercises every decode path, including 0b1000
    under each special value).  Returns (codes [N, K/2] u8, scales [N, K/16]
    u8) as CPU tensors."""
    g = _gen(seed)
    codes = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    if fmt == "weight":
        mag = torch.randint(0, 64 if max_scale_code is None else max_scale_code + 1, (N, K // 16), generator=g, dtype=torch.int32)
        meta = torch.randint(0, 4, (N, K // 16), generator=g, dtype=torch.int32)
        scales = (mag | (meta << 6)).to(torch.uint8)
    else:
        mag = torch.randint(0, 127 if max_scale_code is None else max_scale_code + 1, (N, K // 16), generator=g, dtype=torch.int32)
        meta = torch.randint(0, 2, (N, K // 16), generator=g, dtype=torch.int32) if fmt == "act" else torch.zeros_like(mag)
        scales = (mag | (meta << 7)).to(torch.uint8)
    return codes, scales


def random_packed_variant(N: int, K: int, block: int, scale_fmt: str, n_special: int, *, seed: int = 5):
    """Random packed weights [N, K] of a format variant: uniform code bytes,
    uniform valid scale magnitudes and meta values below n_special.  scale_fmt
    "weight" (E3M3 bytes, meta bits 7..6), "act" / "nvfp4" (E4M3 bytes, meta
    bit 7) or "f16_scale" (16-bit little-endian words: magnitude bits 13..0,
    meta bits 15..14).  Returns (codes [N, K/2] u8, scales [N, K/block] u8 or
    [N, 2 K/block] u8 for the 16-bit words) as CPU tensors."""
    g = _gen(seed)
    codes = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    nb = K // block
    meta = torch.randint(0, max(n_special, 1), (N, nb), generator=g, dtype=torch.int32)
    if scale_fmt == "f16_scale":
        mag = torch.randint(0, 0x4000, (N, nb), generator=g, dtype=torch.int32)
        w = mag | (meta << 14)
        scales = torch.stack([w & 0xFF, w >> 8], dim=2).reshape(N, 2 * nb).to(torch.uint8)
    elif scale_fmt == "weight":
        mag = torch.randint(0, 64, (N, nb), generator=g, dtype=torch.int32)
        scales = (mag | (meta << 6)).to(torch.uint8)
    else:
        mag = torch.randint(0, 127, (N, nb), generator=g, dtype=torch.int32)
        scales = (mag | (meta << 7)).to(torch.uint8)
    return codes, scales
