"""Seeded synthetic inputs for the fused matmul-sample step.

This module only draws inputs: hidden states H [B, d] bf16, LM-head weights
W [V, d] bf16, per-row vocab bitmasks and per-row seeds.  It holds none of the
sampling arithmetic, so both the CUDA path and the CPU oracle may use it.

Trained Qwen3 / Llama heads are not available, so random heads of the same
shapes stand in for them (FlashSampling, arXiv:2603.15854, abstract: decode
workloads on Qwen3-family heads; readus.org page: a vocabulary of about
150k tokens).  Values are normal: H ~ N(0, 1), W ~ N(0, std^2), rounded to
bf16 (round-to-nearest-even by torch).
"""
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

W_SEED = 1234          # generator seed of the weights
H_SEED_BASE = 5678     # generator seed of the hidden states is H_SEED_BASE + B
MASK_SEED = 42         # generator seed of the vocab masks
ROW_SEED_BASE = 1000   # per-row seeds are ROW_SEED_BASE + b


@dataclass(frozen=True)
class Workload:
    """One LM-head workload: shapes, value scales and sampling options."""
    name: str
    d: int
    V: int
    w_std: float
    temperature: float
    batches: Sequence[int]
    per_row_seeds: bool = False
    groups: int = 0                  # 0: flat sampling; G >= 1: grouped
    mask_allowed: Optional[float] = None   # fraction of allowed tokens, None = no mask
    description: str = field(default="", compare=False)


WORKLOADS = {
    "tiny": Workload("tiny", d=256, V=4096, w_std=1.0 / 16.0, temperature=1.0, batches=(1,),
                     description="tiny head, B=1, d=256, V=4096, W ~ N(0, 1/d)"),
    "qwen3-1.7b": Workload("qwen3-1.7b", d=2048, V=151936, w_std=0.02, temperature=1.0,
                           batches=(1, 4, 16, 64),
                           description="Qwen3-1.7B-shaped head, d=2048, V=151936"),
    "qwen3-8b": Workload("qwen3-8b", d=4096, V=151936, w_std=0.02, temperature=0.7,
                         batches=(1, 8, 32, 64, 128, 256), per_row_seeds=True,
                         description="Qwen3-8B-shaped head, d=4096, V=151936, T=0.7, per-row seeds"),
    "large": Workload("large", d=8192, V=128256, w_std=0.015, temperature=1.0,
                      batches=(1, 16, 64, 256),
                      description="large head, d=8192, V=128256 (2.1 GB of weights)"),
    "grouped-masked": Workload("grouped-masked", d=4096, V=151936, w_std=0.02, temperature=0.8,
                               batches=(1, 64, 512), groups=8, mask_allowed=0.5,
                               description="d=4096, V=151936, G=8 contiguous groups, 50% mask"),
}


def _generator(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_hidden(B: int, d: int, device="cpu", seed: Optional[int] = None) -> torch.Tensor:
    """H [B, d] bf16, entries N(0, 1)."""
    seed = H_SEED_BASE + B if seed is None else seed
    g = _generator(device, seed)
    return torch.randn(B, d, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def make_weight(V: int, d: int, std: float, device="cpu", seed: int = W_SEED,
                chunk_rows: int = 16384) -> torch.Tensor:
    """W [V, d] bf16, entries N(0, std^2).  Drawn in row chunks so the fp32
    staging stays small; the chunking is part of the recipe (same seed and
    chunking give the same bytes)."""
    g = _generator(device, seed)
    W = torch.empty(V, d, dtype=torch.bfloat16, device=device)
    for r0 in range(0, V, chunk_rows):
        r1 = min(V, r0 + chunk_rows)
        part = torch.randn(r1 - r0, d, generator=g, device=device, dtype=torch.float32)
        W[r0:r1] = (part * std).to(torch.bfloat16)
    return W


def make_mask(B: int, V: int, allowed: float, device="cpu", seed: int = MASK_SEED) -> torch.Tensor:
    """Per-row vocab bitmask, uint32 words [B, ceil(V/32)] stored as int32.

    Bit (v & 31) of word [b, v >> 5] is 1 when token v is allowed for row b.
    Each token is allowed independently with probability ``allowed``; bits at
    v >= V are 0."""
    g = _generator("cpu", seed)
    words = (V + 31) // 32
    keep = torch.rand(B, words * 32, generator=g) < allowed
    keep[:, V:] = False
    weights = (1 << torch.arange(32, dtype=torch.int64))
    packed = (keep.view(B, words, 32).to(torch.int64) * weights).sum(-1)
    packed = torch.where(packed >= 2 ** 31, packed - 2 ** 32, packed).to(torch.int32)
    return packed.to(device)


def mask_from_bool(allowed: torch.Tensor) -> torch.Tensor:
    """Pack a bool [B, V] allowed-matrix into the uint32 word layout (as int32)."""
    B, V = allowed.shape
    words = (V + 31) // 32
    full = torch.zeros(B, words * 32, dtype=torch.bool)
    full[:, :V] = allowed.cpu()
    weights = (1 << torch.arange(32, dtype=torch.int64))
    packed = (full.view(B, words, 32).to(torch.int64) * weights).sum(-1)
    packed = torch.where(packed >= 2 ** 31, packed - 2 ** 32, packed).to(torch.int32)
    return packed.to(allowed.device)


def make_row_seeds(B: int, device="cpu", base: int = ROW_SEED_BASE) -> torch.Tensor:
    """Per-row seeds base + b, as int64 (read as uint64 by the library)."""
    return (torch.arange(B, dtype=torch.int64) + base).to(device)
