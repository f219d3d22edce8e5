"""The sublayers split across GPUs: one process per GPU, each holding its own
weight shards, with the row-split partial sums reduced over the GPUs.

This is the multi-GPU form of the method ("张量并行：千亿大模型突破单卡显存限制的
底层技术" §2.2 and §3: the MLP's second linear and the attention's output
projection are row-split, so each GPU holds a partial sum of the output and
one AllReduce per sublayer adds them; "TP到底在切什么" §3.3, RowParallelLinear
ends in all_reduce).  Rank r computes its partial sum P_r in the library's
kernels (`tp_mlp_partial_forward` / `tp_attn_partial_forward`), then the
partials are reduced in one of two ways (`mode`):

  "allreduce"  AllReduce of the f32 partial [S, H], then residual + LayerNorm
               on all S rows on every rank.
  "rs_ag"      the AllReduce's two halves ("TP到底在切什么" §5.1: a ring
               AllReduce is a ReduceScatter followed by an AllGather) with the
               LayerNorm in between: ReduceScatter of the partial, so rank r
               holds the sum of rows [r S/N, (r+1) S/N); residual + LayerNorm
               on those S/N rows (the page's remark that the ReduceScatter
               output can be used as it is, split by rows); AllGather of the
               normalised rows into every rank's Y.

The partial sums are reduced in f32 (the pages' "f32 accumulate"); the
AllGather moves the output dtype.  The collectives are torch.distributed calls
(NCCL on GPUs) ordered on the caller's stream; every step of the computation
runs in the library's kernels.
"""
from __future__ import annotations

import contextlib

MODES = ("allreduce", "rs_ag")


def row_split(S: int, world: int, rank: int) -> tuple[int, int]:
    """(first row, row count) of rank's slice of S rows: equal contiguous
    slices, as the ReduceScatter and AllGather of equal-sized tensors give."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside the group")
    if S % world:
        raise ValueError(f"S = {S} rows do not split evenly over {world} ranks")
    rows = S // world
    return rank * rows, rows


class TPSublayer:
    """One rank's part of a sublayer split over `world` GPUs.

    partial(X, P, stream): writes this rank's f32 partial sum P [S, H].
    reduce_ln(rows, parts, X_rows, Y_outs, stream): Y = LN(X + sum(parts)) on
        `rows` rows (tensors starting at the first row), into every output.
    The default reduce_ln is the library's fused reduce + residual + LayerNorm.
    """

    def __init__(self, partial, S: int, H: int, x_dtype, out_dtype, mode: str = "allreduce", group=None,
                 gamma=None, beta=None, eps: float = 1e-5, device=None, reduce_ln=None, world: int | None = None,
                 rank: int | None = None):
        import torch
        import torch.distributed as dist

        if mode not in MODES:
            raise ValueError(f"mode must be one of {MODES}")
        self.partial, self.S, self.H, self.mode, self.group = partial, S, H, mode, group
        self.x_dtype, self.out_dtype = x_dtype, out_dtype
        self.gamma, self.beta, self.eps = gamma, beta, eps
        if world is None:
            world = dist.get_world_size(group) if dist.is_initialized() else 1
        if rank is None:
            rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.world, self.rank = world, rank
        self.P = torch.empty(S, H, dtype=torch.float32, device=device)
        if mode == "rs_ag":
            self.row0, self.rows = row_split(S, world, rank)
            self.P_slice = torch.empty(self.rows, H, dtype=torch.float32, device=device)
            self.Y_slice = torch.empty(self.rows, H, dtype=out_dtype, device=device)
        self.reduce_ln = reduce_ln or self._library_reduce_ln

    def _library_reduce_ln(self, rows, parts, X_rows, Y_outs, stream):
        from . import _lib as L
        L.reduce_residual_layernorm_multi(rows, self.H, parts, X_rows, Y_outs, self.x_dtype, self.out_dtype,
                                          gamma=self.gamma, beta=self.beta, eps=self.eps, stream=stream)

    def forward(self, X, Y, stream=None):
        """Y [S, H] (every rank's copy) = LN(X + sum over ranks of P_r)."""
        import torch
        import torch.distributed as dist

        ctx = torch.cuda.stream(stream) if stream is not None and X.is_cuda else contextlib.nullcontext()
        with ctx:
            self.partial(X, self.P, stream)
            if self.mode == "allreduce":
                if self.world > 1:
                    dist.all_reduce(self.P, group=self.group)
                self.reduce_ln(self.S, [self.P], X, [Y], stream)
            else:
                if self.world > 1:
                    dist.reduce_scatter_tensor(self.P_slice, self.P, group=self.group)
                else:
                    self.P_slice.copy_(self.P)
                r0, n = self.row0, self.rows
                self.reduce_ln(n, [self.P_slice], X[r0:r0 + n], [self.Y_slice], stream)
                if self.world > 1:
                    dist.all_gather_into_tensor(Y, self.Y_slice, group=self.group)
                else:
                    Y.copy_(self.Y_slice)
        return Y


def mlp_partial_fn(A_local, B_local, workspace, act: str = "gelu_tanh"):
    """partial() of the MLP sublayer for the shards this rank holds."""
    from . import _lib as L

    def partial(X, P, stream):
        L.mlp_partial_forward(X, A_local, B_local, P, workspace, act=act, stream=stream)
    return partial


def attn_partial_fn(Wqkv_local, Wo_local, nh_local: int, d: int, workspace):
    """partial() of the attention sublayer for the heads this rank holds."""
    from . import _lib as L

    def partial(X, P, stream):
        L.attn_partial_forward(X, Wqkv_local, Wo_local, nh_local, d, P, workspace, stream=stream)
    return partial
