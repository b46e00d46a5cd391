"""Seeded synthetic workloads and work-unit counts.

This module only draws inputs and counts work.  It holds none of the
attention arithmetic, so both the float64 oracle (through the tests) and the
CUDA path use the same bytes without sharing any computation.

Input recipe (all draws on the CPU with ``torch.Generator().manual_seed``):

* Q, K, V, dO: iid N(0, 1) drawn in float32 in that order, rounded to bf16
  (round to nearest even).
* "peaked" keys: per (batch, head), round(frac * Nk) distinct key positions
  chosen uniformly; those K rows are multiplied by 8 after the bf16 rounding
  (a power of two, so the product is exact in bf16).
* decode: q [B, H, 1, d], K/V caches [B, H, Lmax, d] iid N(0, 1) in bf16 and
  per-sequence lengths L_b drawn uniformly from {lmin, ..., Lmax}; cache slots
  at or beyond L_b hold random data that the kernels must never read.
* FP8 incoherent processing: the random signs s of M = diag(s) H_d / sqrt(d)
  are d independent fair +-1 draws (float32).  "Outlier" inputs scale a few
  whole channels (columns) of Q and K by a power of two after the bf16
  rounding, the situation the rotation is meant for.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = [
    "AttnConfig",
    "DecodeConfig",
    "TINY",
    "C2",
    "SWEEP",
    "LONG",
    "DECODE",
    "make_attention_inputs",
    "make_decode_inputs",
    "make_hadamard_signs",
    "add_outlier_channels",
    "flops_forward",
    "flops_backward",
    "decode_bytes",
]


@dataclass(frozen=True)
class AttnConfig:
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    causal: tuple = (False,)
    seed: int = 0
    peaked_frac: float = 0.0
    peak_factor: float = 8.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    H: int
    Lmax: int
    d: int
    lmin: int
    seed: int = 4

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


# The five workloads: a tiny correctness case, the 2x8x1024x64 case in both
# mask modes, a sequence sweep at 16384 tokens per batch, a 64K-token causal
# case with peaked keys, and ragged split-KV decode.
TINY = AttnConfig("tiny", 1, 2, 128, 128, 64, (False,), seed=0)
C2 = AttnConfig("b2_h8_n1024_d64", 2, 8, 1024, 1024, 64, (True, False), seed=1)
SWEEP = tuple(
    AttnConfig(f"sweep_n{n}_d{d}", 16384 // n, 16, n, n, d, (True,), seed=2)
    for d in (64, 128)
    for n in (512, 1024, 2048, 4096, 8192, 16384)
)
LONG = AttnConfig("long_n65536_d128", 1, 16, 65536, 65536, 128, (True,), seed=3,
                  peaked_frac=0.01, peak_factor=8.0)
DECODE = DecodeConfig("decode_b32_h32_l8192_d128", 32, 32, 8192, 128, 1024, seed=4)


def _randn_bf16(gen: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def make_attention_inputs(B: int, H: int, Nq: int, Nk: int, d: int, seed: int,
                          peaked_frac: float = 0.0, peak_factor: float = 8.0,
                          with_do: bool = True):
    """Return dict(q, k, v, do, peaks) of CPU bf16 tensors [B, H, N, d].

    ``peaks`` is an int64 tensor [B, H, n_peak] of the scaled key positions
    (empty when ``peaked_frac`` is 0).
    """
    gen = torch.Generator().manual_seed(seed)
    q = _randn_bf16(gen, (B, H, Nq, d))
    k = _randn_bf16(gen, (B, H, Nk, d))
    v = _randn_bf16(gen, (B, H, Nk, d))
    do = _randn_bf16(gen, (B, H, Nq, d)) if with_do else None
    n_peak = int(round(peaked_frac * Nk))
    peaks = torch.zeros((B, H, n_peak), dtype=torch.int64)
    if n_peak > 0:
        for b in range(B):
            for h in range(H):
                idx = torch.randperm(Nk, generator=gen)[:n_peak].sort().values
                peaks[b, h] = idx
                k[b, h, idx] = k[b, h, idx] * peak_factor
    return {"q": q, "k": k, "v": v, "do": do, "peaks": peaks}


def make_config_inputs(cfg: AttnConfig, with_do: bool = True):
    return make_attention_inputs(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, cfg.seed,
                                 cfg.peaked_frac, cfg.peak_factor, with_do)


def make_decode_inputs(B: int, H: int, Lmax: int, d: int, lmin: int, seed: int):
    """Return dict(q [B,H,1,d], k_cache, v_cache [B,H,Lmax,d], seqlens int32 [B])."""
    gen = torch.Generator().manual_seed(seed)
    q = _randn_bf16(gen, (B, H, 1, d))
    kc = _randn_bf16(gen, (B, H, Lmax, d))
    vc = _randn_bf16(gen, (B, H, Lmax, d))
    seqlens = torch.randint(lmin, Lmax + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    return {"q": q, "k_cache": kc, "v_cache": vc, "seqlens": seqlens}


def flops_forward(B, H, Nq, Nk, d, causal) -> float:
    """Forward FLOP convention: 4 B H Nq Nk d, halved when causal."""
    f = 4.0 * B * H * Nq * Nk * d
    return f / 2 if causal else f


def flops_backward(B, H, Nq, Nk, d, causal) -> float:
    """Backward FLOP convention: 2.5 x the forward count."""
    return 2.5 * flops_forward(B, H, Nq, Nk, d, causal)


def decode_bytes(seqlens, H: int, d: int, elem_bytes: int = 2) -> int:
    """Algorithmic decode bytes: every visible K and V row read once, plus q and o."""
    total_l = int(torch.as_tensor(seqlens).to(torch.int64).sum())
    B = int(torch.as_tensor(seqlens).numel())
    return total_l * H * d * elem_bytes * 2 + 2 * B * H * d * elem_bytes


def make_hadamard_signs(d: int, seed: int) -> torch.Tensor:
    """d independent fair +-1 draws, float32 (the random diagonal of the incoherent-processing matrix)."""
    gen = torch.Generator().manual_seed(seed)
    return (torch.randint(0, 2, (d,), generator=gen, dtype=torch.int64) * 2 - 1).to(torch.float32)


def add_outlier_channels(x: torch.Tensor, channels, factor: float = 16.0) -> torch.Tensor:
    """Copy of x [..., d] with the given channels multiplied by ``factor`` (a power of two: exact in bf16)."""
    y = x.clone()
    y[..., list(channels)] = y[..., list(channels)] * factor
    return y
