"""Seeded synthetic workloads for fused RoPE + attention and the sin/cos table.

This module only draws inputs: shapes, seeds, random tensors, positions and
sequence lengths.  It holds none of the method's arithmetic (no frequencies,
no trigonometry, no attention) so that the CUDA path and the fp64 oracle can
both take their inputs from it without sharing any computation.

Shapes stand in for the pages' workloads (Qwen-7B-shaped prefill, GQA long
prefill, 16K long context with dynamic NTK, and a packed DynamicNTK batch);
the pages' own model runs need trained weights and are not reproduced.
Recipe: q, k, v ~ N(0, 1) drawn in fp32 with torch.Generator seeded
seed+0/+1/+2, then rounded to bf16 (round-to-nearest-even); positions are
arange per sequence; packed lengths ~ randint(256, 8193) seeded; packed
inverse frequencies ~ U[0, 1) in fp32 seeded seed+3.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    layout: str                 # "BNSD" or "TND"
    B: int                      # batches (BNSD) or packed sequences (TND)
    Hq: int
    Hkv: int
    S: int                      # BNSD sequence length; 0 for TND
    D: int
    rope_base: float = 10000.0
    causal: bool = True
    ntk_train_len: int = 0      # 0: dynamic NTK off
    ntk_factor: float = 1.0
    seed: int = 0
    packed_len_range: tuple = ()  # (lo, hi) for TND lengths ~ randint(lo, hi)
    sincos_dtype: str = "fp16"
    random_inv_freq: bool = False  # TND: invFreq rows drawn ~ U[0,1)
    notes: str = ""


TINY = Workload("tiny B1 H2/2 S128 D64", "BNSD", 1, 2, 2, 128, 64, 10000.0, seed=1, sincos_dtype="fp32")
QWEN7B_PREFILL = Workload("Qwen-7B-shaped prefill B4 H32/32 S2048 D128", "BNSD", 4, 32, 32, 2048, 128, 10000.0,
                          seed=2)
GQA_LONG = Workload("GQA long prefill B2 Hq32 Hkv8 S8192 D128", "BNSD", 2, 32, 8, 8192, 128, 500000.0, seed=3)
NTK_16K = Workload("long context dynamic-NTK B1 Hq64 Hkv8 S16384 D128", "BNSD", 1, 64, 8, 16384, 128, 10000.0,
                   ntk_train_len=8192, ntk_factor=2.0, seed=4)
PACKED = Workload("packed varlen 16 seqs Hq32 Hkv8 D128", "TND", 16, 32, 8, 0, 128, 10000.0, seed=5,
                  packed_len_range=(256, 8193), random_inv_freq=True)

ALL = [TINY, QWEN7B_PREFILL, GQA_LONG, NTK_16K, PACKED]
BY_KEY = {"tiny": TINY, "qwen7b": QWEN7B_PREFILL, "gqa8k": GQA_LONG, "ntk16k": NTK_16K, "packed": PACKED}


def gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


def packed_lengths(w: Workload) -> torch.Tensor:
    lo, hi = w.packed_len_range
    return torch.randint(lo, hi, (w.B,), generator=gen(w.seed), dtype=torch.int32)


def seq_lengths(w: Workload) -> List[int]:
    if w.layout == "TND":
        return [int(x) for x in packed_lengths(w)]
    return [w.S] * w.B


def ntokens(w: Workload) -> int:
    return sum(seq_lengths(w))


def randn16(shape, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    return torch.randn(*shape, generator=gen(seed), dtype=torch.float32).to(dtype)


def make_qkv(w: Workload, dtype=torch.bfloat16):
    """q, k, v on the CPU in w's layout."""
    if w.layout == "BNSD":
        qs, ks = (w.B, w.Hq, w.S, w.D), (w.B, w.Hkv, w.S, w.D)
    else:
        T = ntokens(w)
        qs, ks = (T, w.Hq, w.D), (T, w.Hkv, w.D)
    return randn16(qs, w.seed + 0, dtype), randn16(ks, w.seed + 1, dtype), randn16(ks, w.seed + 2, dtype)


def positions(w: Workload) -> torch.Tensor:
    """BNSD: [B, S] arange per batch.  TND: [T] concatenated aranges."""
    if w.layout == "BNSD":
        return torch.arange(w.S, dtype=torch.int32).repeat(w.B, 1).contiguous()
    return torch.cat([torch.arange(n, dtype=torch.int32) for n in seq_lengths(w)])


def random_inv_freq(w: Workload) -> Optional[torch.Tensor]:
    """Drawn per-sequence inverse frequencies [B, D/2] in [0, 1), or None."""
    if not w.random_inv_freq:
        return None
    return torch.rand(w.B, w.D // 2, generator=gen(w.seed + 3), dtype=torch.float32)


def sincos_problem(T: int, D: int, batch: int, seed: int):
    """A sin/cos-table input: positionIds [T], invFreq [batch, D/2] in [0,1),
    seqLens [batch] (positive, summing to T, near-equal split)."""
    base, extra = divmod(T, batch)
    lens = torch.tensor([base + (1 if b < extra else 0) for b in range(batch)], dtype=torch.int32)
    pos = torch.cat([torch.arange(int(n), dtype=torch.int32) for n in lens])
    inv = torch.rand(batch, D // 2, generator=gen(seed), dtype=torch.float32)
    return pos, inv, lens
