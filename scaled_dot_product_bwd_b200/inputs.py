"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds none of the attention arithmetic: it only draws random
tensors.  Recipe: one ``torch.Generator`` seeded with ``seed``; float32
N(0, 1) draws in the order Q, K, V, dO, then the T5 table or the dense bias;
Q, K, V and dO are rounded to bfloat16 (round-to-nearest-even), the bias and
table stay float32.  Everything is generated on the CPU so that both sides of
a parity check see the same values.

Layouts: Q, dO [B, L, Hq, d]; K, V [B, Lk, Hkv, d] (batch, sequence, heads,
head dim -- the (B, T, N, H) layout of the codelab "jax-gpu-05-attention-gpu",
section 3); T5 table [num_buckets, Hq]; dense bias [B, Hq, L, Lk]; ALiBi
slopes [Hq].  Packed variable-length batches draw one sequence axis
(B = 1) and are cut by cumulative lengths (``cu_seqlens``).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass
class Inputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    do: torch.Tensor
    t5_table: torch.Tensor | None = None
    bias: torch.Tensor | None = None
    alibi_slopes: torch.Tensor | None = None
    rel_table: torch.Tensor | None = None


def make_inputs(B: int, L: int, Hq: int, Hkv: int, d: int, *, seed: int = 0,
                t5_buckets: int = 0, dense_bias: bool = False,
                bias_shape: tuple | None = None, alibi: bool = False,
                Lk: int | None = None, rel_table: bool = False) -> Inputs:
    """Draw Q, K, V, dO (bf16) and optionally a T5 table / dense bias (fp32).

    K and V have Lk rows (default L).  A relative-position table is
    [L + Lk - 1, Hq] N(0,1) fp32, drawn last.  ALiBi slopes are not drawn: they are
    the geometric sequence of Press et al. 2022, 2^(-8 (h + 1) / Hq) for head
    h (fp32)."""
    g = torch.Generator().manual_seed(seed)
    Lk = L if Lk is None else Lk

    def randn(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32)

    q = randn(B, L, Hq, d).to(torch.bfloat16)
    k = randn(B, Lk, Hkv, d).to(torch.bfloat16)
    v = randn(B, Lk, Hkv, d).to(torch.bfloat16)
    do = randn(B, L, Hq, d).to(torch.bfloat16)
    table = randn(t5_buckets, Hq) if t5_buckets else None
    bias = None
    if dense_bias:
        bias = randn(*(bias_shape or (B, Hq, L, Lk)))
    slopes = None
    if alibi:
        slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / Hq) for h in range(Hq)],
                              dtype=torch.float32)
    rel = randn(L + Lk - 1, Hq) if rel_table else None
    return Inputs(q, k, v, do, table, bias, slopes, rel)


def make_fire_params(width: int, heads: int, *, seed: int = 0) -> dict:
    """Seeded FIRE MLP weights (fp32): w1, b1 [width] ~ N(0,1) and N(0,1) / 2,
    w2 [heads, width] ~ N(0,1) / sqrt(width), b2 [heads] ~ N(0,1) / 2."""
    g = torch.Generator().manual_seed(seed)

    def randn(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32)

    return dict(w1=randn(width), b1=randn(width) * 0.5,
                w2=randn(heads, width) * (1.0 / width ** 0.5), b2=randn(heads) * 0.5)


# The workloads of the benchmark table, by name.  Each entry: shapes, mask and
# bias.  window_left follows the inclusive reading i - w <= j <= i.
WORKLOADS = {
    "tiny": dict(B=1, Hq=2, Hkv=2, L=128, d=64, causal=True, window_left=-1, bias="none"),
    "mistral4k": dict(B=4, Hq=32, Hkv=8, L=4096, d=128, causal=True, window_left=4096, bias="none"),
    "mistral8k": dict(B=2, Hq=32, Hkv=8, L=8192, d=128, causal=True, window_left=4096, bias="none"),
    "t5rpe": dict(B=16, Hq=12, Hkv=12, L=1024, d=64, causal=False, window_left=-1, bias="t5"),
    "t5dense": dict(B=16, Hq=12, Hkv=12, L=1024, d=64, causal=False, window_left=-1, bias="dense"),
}


def cu_seqlens(lengths) -> torch.Tensor:
    """Cumulative offsets [0, l0, l0 + l1, ...] (int32) of packed sequences."""
    out = [0]
    for n in lengths:
        out.append(out[-1] + int(n))
    return torch.tensor(out, dtype=torch.int32)
