"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and names the workloads.  It holds none
of the method's arithmetic, so both the CUDA path and the CPU oracle may use it
without sharing any computation.

Every tensor is drawn on the CPU from ``torch.Generator().manual_seed(seed)``
as float32 standard normals, scaled, then cast to the workload's dtype; the
same bits are copied to the GPU and handed to the oracle.  Draw order for a
prefill workload is q, then k, then v.  A decode workload draws its initial
state from ``seed`` and the q, k, v of step i from ``seed + 1 + i``.

The shapes follow the model the pages describe: head dim 128, 128 query heads
sharing 32 kv heads ("MiniMax-01与Lightning Attention", section 1.1), contexts
up to a million tokens.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Prefill:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    chunks: tuple
    dtype: torch.dtype
    seed: int
    qk_scale: float = 1.0      # multiplies N(0,1)/sqrt(d) for q and k
    v_over_sqrt_d: bool = False  # v ~ N(0,1)/sqrt(d) instead of N(0,1)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def describe(self) -> str:
        vs = "N(0,1)/sqrt(d)" if self.v_over_sqrt_d else "N(0,1)"
        qs = "N(0,1)/sqrt(d)" + (f"*{self.qk_scale:g}" if self.qk_scale != 1.0 else "")
        return (f"B={self.B} Hq={self.Hq} Hkv={self.Hkv} N={self.N} d={self.d} "
                f"chunk={'|'.join(map(str, self.chunks))} {str(self.dtype).split('.')[-1]}; "
                f"q,k ~ {qs}; v ~ {vs}; seed {self.seed}")


@dataclass(frozen=True)
class Decode:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    steps: int
    seed: int
    dtype: torch.dtype = torch.bfloat16

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


# The five workloads, named by what they are.
PR1_F32 = Prefill("causal-f32 B1 H2 N1024 d64", 1, 2, 2, 1024, 64, (64,), torch.float32, 0,
                  v_over_sqrt_d=True)
MHA_8K = Prefill("mha B4 H16 N8192 d128", 4, 16, 16, 8192, 128, (64,), torch.bfloat16, 1)
GQA_32K = Prefill("gqa B1 Hq128/Hkv32 N32768 d128", 1, 128, 32, 32768, 128, (64, 128),
                  torch.bfloat16, 2)
LONG_1M = Prefill("long B1 H8 N1048576 d128", 1, 8, 8, 1 << 20, 128, (128,), torch.bfloat16, 3,
                  qk_scale=0.5)
DECODE_B256 = Decode("decode B256 Hq64/Hkv16 d128", 256, 64, 16, 128, 64, 4)

PREFILL_WORKLOADS = (PR1_F32, MHA_8K, GQA_32K, LONG_1M)


def _randn(gen: torch.Generator, shape, scale: float, dtype: torch.dtype) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


def prefill_inputs(w: Prefill, N: int | None = None, B: int | None = None,
                   Hq: int | None = None, Hkv: int | None = None, seed: int | None = None):
    """q [B,Hq,N,d], k, v [B,Hkv,N,d] on the CPU, drawn as the workload states.

    N, B, Hq, Hkv and seed may be overridden to make a smaller case of the same
    distribution (the parity tests use this)."""
    B = w.B if B is None else B
    Hq = w.Hq if Hq is None else Hq
    Hkv = w.Hkv if Hkv is None else Hkv
    N = w.N if N is None else N
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    s = 1.0 / math.sqrt(w.d)
    q = _randn(gen, (B, Hq, N, w.d), s * w.qk_scale, w.dtype)
    k = _randn(gen, (B, Hkv, N, w.d), s * w.qk_scale, w.dtype)
    v = _randn(gen, (B, Hkv, N, w.d), s if w.v_over_sqrt_d else 1.0, w.dtype)
    return q, k, v


def random_qkv(B: int, Hq: int, Hkv: int, N: int, d: int, dtype: torch.dtype, seed: int,
               qk_scale: float | None = None, v_scale: float = 1.0):
    """Arbitrary-shape q, k, v with the same recipe (q,k ~ N(0,1)/sqrt(d), v ~ N(0,1))."""
    gen = torch.Generator().manual_seed(seed)
    s = (1.0 / math.sqrt(d)) if qk_scale is None else qk_scale
    q = _randn(gen, (B, Hq, N, d), s, dtype)
    k = _randn(gen, (B, Hkv, N, d), s, dtype)
    v = _randn(gen, (B, Hkv, N, d), v_scale, dtype)
    return q, k, v


def decode_state(w: Decode, B: int | None = None) -> torch.Tensor:
    """Initial fp32 state S [B,Hkv,d,d] ~ N(0,1)/d."""
    B = w.B if B is None else B
    gen = torch.Generator().manual_seed(w.seed)
    return _randn(gen, (B, w.Hkv, w.d, w.d), 1.0 / w.d, torch.float32)


def decode_token(w: Decode, step: int, B: int | None = None):
    """q [B,Hq,d], k, v [B,Hkv,d] for decode step ``step``."""
    B = w.B if B is None else B
    gen = torch.Generator().manual_seed(w.seed + 1 + step)
    s = 1.0 / math.sqrt(w.d)
    q = _randn(gen, (B, w.Hq, w.d), s, w.dtype)
    k = _randn(gen, (B, w.Hkv, w.d), s, w.dtype)
    v = _randn(gen, (B, w.Hkv, w.d), 1.0, w.dtype)
    return q, k, v
