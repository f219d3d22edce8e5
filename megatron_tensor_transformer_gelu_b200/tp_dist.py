"""The sublayers split across GPUs: one process per GPU, each holding its own
weight shards, with the row-split partial sums reduced over the GPUs.

This is the multi-GPU form of the method ("张量并行：千亿大模型突破单卡显存限制的
底层技术" §2.2 and §3: the MLP's second linear and the attention's output
projection are row-split, so each GPU holds a partial sum of the output and
one AllReduce per sublayer adds them; "TP到底在切什么" §3.3, RowParallelLinear
ends in all_reduce).  Rank r computes its partial sum P_r in the library's
kernels (`tp_mlp_partial_forward` / `tp_attn_partial_forward`), then the
partials are reduced in one of three ways (`mode`):

  "allreduce"  AllReduce of the f32 partial [S, H], then residual + LayerNorm
               on all S rows on every rank.
  "rs_ag"      the AllReduce's two halves ("TP到底在切什么" §5.1: a ring
               AllReduce is a ReduceScatter followed by an AllGather) with the
               LayerNorm in between: ReduceScatter of the partial, so rank r
               holds the sum of rows [r S/N, (r+1) S/N); residual + LayerNorm
               on those S/N rows (the page's remark that the ReduceScatter
               output can be used as it is, split by rows); AllGather of the
               normalised rows into every rank's Y.
  "peer"       the same three steps in one kernel over peer memory: every
               rank's partial and output buffer are mapped into every rank's
               process (CUDA IPC); after a device-side barrier (every partial
               complete), rank r's kernel reads its S/N rows from every rank's
               partial (peer loads), normalises them and stores them into every
               rank's output (peer stores); a second barrier orders those
               stores before any rank reads its output.

The partial sums are reduced in f32 (the pages' "f32 accumulate"); the
AllGather moves the output dtype.  The collectives are torch.distributed calls
(NCCL on GPUs) ordered on the caller's stream; every step of the computation
runs in the library's kernels.
"""
from __future__ import annotations

import contextlib

MODES = ("allreduce", "rs_ag", "peer")


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
                 rank: int | None = None, peer_ops=None, exchange=None):
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
        self._imported = []
        if mode == "peer":
            self._setup_peer(out_dtype, device, peer_ops, exchange)

    def _setup_peer(self, out_dtype, device, peer_ops, exchange):
        """Map every rank's partial, output buffer and barrier flags into this
        process.  peer_ops: export / import_ / close / barrier (default: the
        library's CUDA IPC entry points and device barrier); exchange(obj) ->
        every rank's obj (default: torch.distributed.all_gather_object)."""
        import torch
        import torch.distributed as dist

        self.ops = peer_ops or _LibraryPeerOps()
        self.row0, self.rows = row_split(self.S, self.world, self.rank)
        self.Ybuf = torch.empty(self.S, self.H, dtype=out_dtype, device=device)
        self.flags = torch.zeros(self.world, dtype=torch.int64, device=device)
        self.epoch = 0
        mine = (self.ops.export(self.P), self.ops.export(self.Ybuf), self.ops.export(self.flags))
        if exchange is None:
            def exchange(obj):
                if self.world == 1:
                    return [obj]
                out = [None] * self.world
                dist.all_gather_object(out, obj, group=self.group)
                return out
        every = exchange(mine)
        self.P_addr, self.Y_addr, self.F_addr = [], [], []
        for q in range(self.world):
            if q == self.rank:
                addrs = (self.P.data_ptr(), self.Ybuf.data_ptr(), self.flags.data_ptr())
            else:
                addrs = tuple(self.ops.import_(h) for h in every[q])
                self._imported.extend(addrs)
            self.P_addr.append(addrs[0])
            self.Y_addr.append(addrs[1])
            self.F_addr.append(addrs[2])

    def close(self):
        """Unmap the other ranks' buffers (peer mode)."""
        for a in self._imported:
            self.ops.close(a)
        self._imported = []

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
            elif self.mode == "peer":
                r0, n = self.row0, self.rows
                yb = self.Ybuf.element_size()
                self.epoch += 1
                self.ops.barrier(self.world, self.rank, self.F_addr, self.epoch, stream)
                self.reduce_ln(n, [a + r0 * self.H * 4 for a in self.P_addr], X[r0:r0 + n],
                               [a + r0 * self.H * yb for a in self.Y_addr], stream)
                self.epoch += 1
                self.ops.barrier(self.world, self.rank, self.F_addr, self.epoch, stream)
                if Y.data_ptr() != self.Ybuf.data_ptr():
                    Y.copy_(self.Ybuf)
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


class _LibraryPeerOps:
    """The library's CUDA IPC entry points and device-side barrier."""

    @staticmethod
    def export(t):
        from . import _lib as L
        return L.ipc_export(t)

    @staticmethod
    def import_(handle):
        from . import _lib as L
        return L.ipc_import(handle)

    @staticmethod
    def close(addr):
        from . import _lib as L
        L.ipc_close(addr)

    @staticmethod
    def barrier(nranks, rank, flag_addrs, epoch, stream):
        from . import _lib as L
        L.peer_barrier(nranks, rank, flag_addrs, epoch, stream=stream)


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
