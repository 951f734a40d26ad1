"""Seeded synthetic inputs for every workload of the block-scaled FP4 path.

This module only draws random tensors (torch's generator, fixed seeds) and builds
MoE routing offsets.  It holds none of the FP4 method's arithmetic, so both the
CPU oracle and the CUDA path can be fed from it without sharing code.

Recipes (shapes follow the pages' LLM inference and training workloads):
  * glossary experiment: ``torch.manual_seed(0); x = randn(4096); x[::512] *= 20``
    (the "FP4" glossary entry's block-size experiment, ultralytics.com).
  * pr1: A, B = randn(512, 512) (seed 0, A drawn first), flat every 512th element x20.
  * decode: W [28672, 8192] ~ N(0, 0.02) fp32 (seed 1); X [16, 8192] bf16 ~ N(0, 1)
    with 0.1% of elements (positions from randperm) multiplied by 50 (seed 2).
  * prefill: X [8192, 8192] bf16 N(0,1) + 0.1% x50 (seed 3); W [8192, 8192]
    N(0, 0.02) (seed 4).
  * moe: 4096 tokens, 32 experts, top-4 of uniform gates rand(4096, 32) (seed 5);
    the 16384 (token, expert) rows sorted by expert (stable) give offsets[33];
    A [16384, 2880] bf16 N(0,1) + 0.1% x50 (seed 6); W [32, 5760, 2880] N(0, 0.02)
    fp32 (seed 7).
  * train S: W [S, S] fp32 N(0, 0.02) (seed 8); X, dY [S, S] bf16 N(0, 1)
    (seeds 9, 10).
"""
from __future__ import annotations

import torch

__all__ = [
    "glossary_experiment_input", "pr1_inputs", "normal", "with_outliers", "decode_inputs",
    "prefill_inputs", "moe_routing", "moe_inputs", "train_inputs", "bf16_bits",
]


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def glossary_experiment_input() -> torch.Tensor:
    """4096 N(0,1) values from torch's CPU generator at seed 0, every 512th x20."""
    torch.manual_seed(0)
    x = torch.randn(4096)
    x[::512] *= 20
    return x


def pr1_inputs():
    """A, B [512, 512] fp32 N(0,1) at seed 0 (A first), every 512th element x20."""
    g = _gen(0)
    a = torch.randn(512, 512, generator=g)
    b = torch.randn(512, 512, generator=g)
    a.view(-1)[::512] *= 20
    b.view(-1)[::512] *= 20
    return a, b


def normal(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(*shape, generator=g, device=device) * std


def with_outliers(x: torch.Tensor, seed: int, frac: float = 0.001, factor: float = 50.0) -> torch.Tensor:
    """Multiply round(frac * n) randomly chosen elements by ``factor`` (in place)."""
    n = x.numel()
    count = int(round(frac * n))
    g = _gen(seed + 1000, x.device)
    idx = torch.randperm(n, generator=g, device=x.device)[:count]
    x.view(-1)[idx] *= factor
    return x


def decode_inputs(device="cpu", m: int = 16, n: int = 28672, k: int = 8192):
    w = normal((n, k), 0.02, 1, device)
    x = with_outliers(normal((m, k), 1.0, 2, device), 2).to(torch.bfloat16)
    return x, w


def prefill_inputs(device="cpu", m: int = 8192, n: int = 8192, k: int = 8192):
    x = with_outliers(normal((m, k), 1.0, 3, device), 3).to(torch.bfloat16)
    w = normal((n, k), 0.02, 4, device)
    return x, w


def moe_routing(tokens: int = 4096, experts: int = 32, topk: int = 4, seed: int = 5):
    """Top-k of uniform gates; returns (token index per row sorted by expert, offsets)."""
    g = _gen(seed)
    gates = torch.rand(tokens, experts, generator=g)
    top = torch.topk(gates, topk, dim=1).indices            # [tokens, topk]
    expert_of_row = top.reshape(-1)                          # row = token * topk + j
    order = torch.sort(expert_of_row, stable=True).indices   # group rows by expert
    token_of_row = order // topk
    counts = torch.bincount(expert_of_row, minlength=experts)
    offsets = torch.zeros(experts + 1, dtype=torch.int32)
    offsets[1:] = torch.cumsum(counts, 0).to(torch.int32)
    return token_of_row, offsets


def moe_inputs(device="cpu", tokens: int = 4096, experts: int = 32, topk: int = 4,
               n: int = 5760, k: int = 2880):
    token_of_row, offsets = moe_routing(tokens, experts, topk)
    rows = tokens * topk
    a = with_outliers(normal((rows, k), 1.0, 6, device), 6).to(torch.bfloat16)
    w = normal((experts, n, k), 0.02, 7, device)
    return a, w, offsets, token_of_row


def train_inputs(s: int, device="cpu"):
    w = normal((s, s), 0.02, 8, device)
    x = normal((s, s), 1.0, 9, device).to(torch.bfloat16)
    dy = normal((s, s), 1.0, 10, device).to(torch.bfloat16)
    return x, w, dy


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (how the oracle takes bf16 input)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
