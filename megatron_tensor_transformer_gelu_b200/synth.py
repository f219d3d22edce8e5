"""Seeded synthetic inputs for the tensor-parallel Transformer sublayer.

This module is shared by the CUDA path's tests/bench and by the oracle's tests.
It holds no arithmetic of the method: it only draws random numbers, casts them
to the storage type, cuts full matrices into contiguous shards (pure data
movement) and picks the row sample that parity checks compare.

Recipe (one generator per workload, drawn in a fixed order):
  * ``torch.Generator().manual_seed(seed)`` on the CPU;
  * X ~ N(0, 1); first-layer weight ~ N(0, 1/fan_in); second-layer weight
    ~ N(0, 1/fan_in), fan_in being the weight's number of rows; the
    "N(0, 1/fan_in)" of the pages' linear layers ("TP 到底在切什么" page, §3.2
    ColumnParallelLinear / §3.3 RowParallelLinear: ``randn(out, in) / sqrt(in)``)
    is read as variance 1/fan_in, i.e. standard deviation 1/sqrt(fan_in);
  * values are drawn in fp32 and then rounded (round-to-nearest-even) to the
    workload's storage type, so both sides see exactly the same numbers.

Shard layout: each shard is its own contiguous buffer, as the pages' weight
chunking does (``narrow(dim, rank*chunk, chunk).clone()``, "TP 到底在切什么"
page §3.1).  Column shards of a ``[in, out]`` weight take ``out/t`` consecutive
columns; row shards take ``in/t`` consecutive rows.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

__all__ = [
    "MlpInputs", "AttnInputs", "LinearInputs",
    "gen_mlp", "gen_attn", "gen_linear",
    "split_columns", "split_rows", "split_qkv_by_head", "split_rows_by_head",
    "row_sample",
]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


@dataclass
class MlpInputs:
    X: torch.Tensor      # [S, H]
    A: torch.Tensor      # [H, F]  first (expansion) weight, pages' [in, out] layout
    B: torch.Tensor      # [F, H]  second (compression) weight
    gamma: torch.Tensor  # [H] f32
    beta: torch.Tensor   # [H] f32


@dataclass
class AttnInputs:
    X: torch.Tensor      # [S, H]
    Wqkv: torch.Tensor   # [H, 3H] = [W_Q | W_K | W_V], head j in columns j*d.. of each block
    Wo: torch.Tensor     # [H, H]
    gamma: torch.Tensor
    beta: torch.Tensor


@dataclass
class LinearInputs:
    X: torch.Tensor      # [M, K]
    W: torch.Tensor      # [K, N]


def _weights(g, rows, cols, dtype):
    return (torch.randn(rows, cols, generator=g) / math.sqrt(rows)).to(dtype)


def gen_mlp(S: int, H: int, F: int, seed: int = 0, dtype=torch.bfloat16) -> MlpInputs:
    g = _gen(seed)
    X = torch.randn(S, H, generator=g).to(dtype)
    A = _weights(g, H, F, dtype)
    B = _weights(g, F, H, dtype)
    return MlpInputs(X, A, B, torch.ones(H), torch.zeros(H))


def gen_attn(S: int, H: int, seed: int = 0, dtype=torch.bfloat16) -> AttnInputs:
    g = _gen(seed)
    X = torch.randn(S, H, generator=g).to(dtype)
    Wqkv = _weights(g, H, 3 * H, dtype)
    Wo = _weights(g, H, H, dtype)
    return AttnInputs(X, Wqkv, Wo, torch.ones(H), torch.zeros(H))


def gen_linear(M: int, K: int, N: int, seed: int = 0, dtype=torch.bfloat16) -> LinearInputs:
    g = _gen(seed)
    X = torch.randn(M, K, generator=g).to(dtype)
    W = _weights(g, K, N, dtype)
    return LinearInputs(X, W)


def gen_upstream(S: int, H: int, seed: int = 0, dtype=torch.bfloat16):
    """Upstream gradient dY ~ N(0, 1) [S, H] and a LayerNorm scale gamma ~
    1 + N(0, 1)/4, beta ~ N(0, 1)/4 (f32 [H]) for backward tests: the same
    recipe as the forward inputs, from its own seeded generator."""
    g = _gen(seed)
    dY = torch.randn(S, H, generator=g).to(dtype)
    gamma = 1.0 + 0.25 * torch.randn(H, generator=g)
    beta = 0.25 * torch.randn(H, generator=g)
    return dY, gamma, beta


def split_columns(W: torch.Tensor, t: int) -> list[torch.Tensor]:
    """t contiguous column shards of a [in, out] matrix."""
    n = W.shape[1]
    assert n % t == 0, "shard count must divide the column count"
    c = n // t
    return [W[:, i * c:(i + 1) * c].contiguous() for i in range(t)]


def split_rows(W: torch.Tensor, t: int) -> list[torch.Tensor]:
    """t contiguous row shards of a [in, out] matrix."""
    n = W.shape[0]
    assert n % t == 0, "shard count must divide the row count"
    r = n // t
    return [W[i * r:(i + 1) * r, :].contiguous() for i in range(t)]


def split_qkv_by_head(Wqkv: torch.Tensor, nh: int, d: int, t: int) -> list[torch.Tensor]:
    """Shard s holds heads [s*nh/t, (s+1)*nh/t) of each of the Q, K and V blocks,
    concatenated as [Q_s | K_s | V_s] (each block nh/t*d columns)."""
    H = nh * d
    assert Wqkv.shape[1] == 3 * H and nh % t == 0
    w = (nh // t) * d
    out = []
    for s in range(t):
        cols = [Wqkv[:, blk * H + s * w: blk * H + (s + 1) * w] for blk in range(3)]
        out.append(torch.cat(cols, dim=1).contiguous())
    return out


def split_rows_by_head(Wo: torch.Tensor, nh: int, d: int, t: int) -> list[torch.Tensor]:
    """O-projection shard s: the rows that multiply shard s's heads."""
    return split_rows(Wo, t)


def row_sample(S: int, seed: int, n: int = 64) -> list[int]:
    """Deterministic sample of output rows: 0, S-1 and n-2 rows drawn with ``seed``."""
    if S <= n:
        return list(range(S))
    g = _gen(seed)
    picks = {0, S - 1}
    perm = torch.randperm(S - 2, generator=g)[: n - 2] + 1
    picks.update(int(i) for i in perm)
    return sorted(picks)
