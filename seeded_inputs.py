"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws random numbers and rounds them to the storage type the
workload names. It holds none of the attention or merge arithmetic, so both the
CUDA path and the CPU oracle can consume its tensors without sharing any of the
method's code.

Recipe (one CPU ``torch.Generator`` per call, seeded):

* attention workloads draw ``randn`` fp32 in the order Q, K, V with shapes
  ``[B, S, Hq, D]``, ``[B, S, Hkv, D]``, ``[B, S, Hkv, D]``; bf16 workloads
  round each tensor to bf16 (round-to-nearest-even) right after drawing it.
  Tensors above ``CHUNK_ROWS`` tokens are drawn in consecutive token chunks of
  ``CHUNK_ROWS`` from the same generator, so that a 1M-token draw never holds
  more than one fp32 chunk at a time.
* backward inputs draw Q, K, V as the attention workloads do, then the
  upstream gradient dO ``[B, S, Hq, D]`` ``randn`` from the same generator,
  rounded like Q.
* decode workloads draw ``q`` ``[B, Tq, Hq, D]``, then the cache ``k``, ``v``
  ``[B, Skv, Hkv, D]``, ``randn`` rounded to bf16, in that order.
* merge workloads draw, for partial i = 0..k-1 in turn, ``out_i`` ~ N(0, 1) of
  ``[T, H, D]`` fp32 and then ``lse_i`` ~ U(-5, 15) of ``[T, H]`` fp32
  (``rand * 20 - 5``).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

CHUNK_ROWS = 65536


@dataclass(frozen=True)
class AttnWorkload:
    """Shape of one blockwise-attention workload (names follow the pages)."""

    name: str
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    n_blocks: int
    causal: bool
    partition: str  # "contiguous" or "zigzag"
    in_dtype: str  # "f32" or "bf16"
    out_dtype: str  # "f32" or "bf16"

    @property
    def gqa_groups(self) -> int:
        return self.Hq // self.Hkv

    @property
    def visible_pairs(self) -> int:
        """(query, key) pairs inside the mask, per (batch, query head)."""
        S = self.S
        return S * (S + 1) // 2 if self.causal else S * S

    @property
    def flops(self) -> float:
        """Causal-adjusted algorithmic FLOPs: QK^T and PV, 2 flops per MAC."""
        return 4.0 * self.B * self.Hq * self.D * self.visible_pairs


# The five workloads: the tiny exactness case, the 4k zigzag case, the 24k
# GQA case shaped like the TokenRing per-step profile, the merge sweep (below)
# and the 1M-token long-context case.
WORKLOADS = {
    "tiny": AttnWorkload("tiny", 1, 256, 2, 2, 64, 4, False, "contiguous", "f32", "f32"),
    "zigzag4k": AttnWorkload("zigzag4k", 1, 4096, 8, 8, 128, 4, True, "zigzag", "bf16", "f32"),
    "gqa24k": AttnWorkload("gqa24k", 1, 24000, 32, 8, 128, 4, True, "zigzag", "bf16", "f32"),
    "long1m": AttnWorkload("long1m", 1, 1048576, 8, 2, 128, 8, True, "zigzag", "bf16", "bf16"),
}


@dataclass(frozen=True)
class DecodeWorkload:
    """Decode phase: the last Tq tokens against a cache of Skv tokens."""

    name: str
    B: int
    Tq: int
    Skv: int
    Hq: int
    Hkv: int
    D: int
    causal: bool
    out_dtype: str  # "f32" or "bf16"

    @property
    def gqa_groups(self) -> int:
        return self.Hq // self.Hkv

    @property
    def bytes(self) -> int:
        """Bytes one call must move: the K and V cache and Q read (bf16), out
        written and lse (fp32) written."""
        ob = 4 if self.out_dtype == "f32" else 2
        rows = self.B * self.Tq * self.Hq
        return 2 * 2 * self.B * self.Skv * self.Hkv * self.D + rows * self.D * (2 + ob) + rows * 4


# Decode against the long-context cache (one token, the 1M-token GQA shape)
# and a batch of sequences shaped like the 24k profile with four tokens each.
DECODE_WORKLOADS = {
    "decode1m": DecodeWorkload("decode1m", 1, 1, 1048576, 8, 2, 128, True, "f32"),
    "decode24k": DecodeWorkload("decode24k", 8, 4, 24000, 32, 8, 128, True, "f32"),
}

MERGE_HEADS = 32
MERGE_DIM = 128
MERGE_TOKENS = [4096 * 2 ** i for i in range(9)]  # 4,096 ... 1,048,576
MERGE_PARTIALS = [2, 4, 8, 16]


def _draw(gen: torch.Generator, shape, dtype: torch.dtype) -> torch.Tensor:
    B, S = shape[0], shape[1]
    out = torch.empty(shape, dtype=dtype)
    for b in range(B):
        for s0 in range(0, S, CHUNK_ROWS):
            s1 = min(S, s0 + CHUNK_ROWS)
            x = torch.randn((s1 - s0,) + tuple(shape[2:]), generator=gen, dtype=torch.float32)
            out[b, s0:s1] = x.to(dtype)
    return out


def attention_inputs(B: int, S: int, Hq: int, Hkv: int, D: int, dtype: str = "bf16",
                     seed: int = 0):
    """Q, K, V on the host, drawn in that order from one generator."""
    tdt = {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]
    gen = torch.Generator("cpu").manual_seed(seed)
    q = _draw(gen, (B, S, Hq, D), tdt)
    k = _draw(gen, (B, S, Hkv, D), tdt)
    v = _draw(gen, (B, S, Hkv, D), tdt)
    return q, k, v


def backward_inputs(B: int, S: int, Hq: int, Hkv: int, D: int, dtype: str = "bf16", seed: int = 0):
    """Q, K, V (as ``attention_inputs``) and then dO, from one generator."""
    tdt = {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]
    gen = torch.Generator("cpu").manual_seed(seed)
    q = _draw(gen, (B, S, Hq, D), tdt)
    k = _draw(gen, (B, S, Hkv, D), tdt)
    v = _draw(gen, (B, S, Hkv, D), tdt)
    do = _draw(gen, (B, S, Hq, D), tdt)
    return q, k, v, do


def decode_inputs(B: int, Tq: int, Skv: int, Hq: int, Hkv: int, D: int, seed: int = 0):
    """q [B, Tq, Hq, D], then the cache k, v [B, Skv, Hkv, D], bf16, drawn in
    that order from one generator."""
    gen = torch.Generator("cpu").manual_seed(seed)
    q = _draw(gen, (B, Tq, Hq, D), torch.bfloat16)
    k = _draw(gen, (B, Skv, Hkv, D), torch.bfloat16)
    v = _draw(gen, (B, Skv, Hkv, D), torch.bfloat16)
    return q, k, v


def workload_inputs(w: AttnWorkload, seed: int = 0):
    return attention_inputs(w.B, w.S, w.Hq, w.Hkv, w.D, w.in_dtype, seed)


def merge_inputs(T: int, k: int, H: int = MERGE_HEADS, D: int = MERGE_DIM, seed: int = 0):
    """k partials (out_i, lse_i): out ~ N(0,1) [T,H,D] fp32, lse ~ U(-5,15) [T,H] fp32."""
    gen = torch.Generator("cpu").manual_seed(seed)
    outs, lses = [], []
    for _ in range(k):
        outs.append(torch.randn((T, H, D), generator=gen, dtype=torch.float32))
        lses.append(torch.rand((T, H), generator=gen, dtype=torch.float32) * 20.0 - 5.0)
    return outs, lses
