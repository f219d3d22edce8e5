"""The multi-GPU sublayer's host logic on CPU: world-size 2 and 4 gloo ranks
run tp_dist.TPSublayer with stub partials and a stub reduction (Y = X + the
sum of the partials, no LayerNorm), so the row bookkeeping of both reduction
modes is checked without a GPU: the AllReduce form, and the ReduceScatter ->
per-slice reduction -> AllGather form.  Every rank must end with the same Y,
equal to X plus every rank's partial, and each rank's slice reduction must see
exactly its own rows."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from megatron_tensor_transformer_gelu_b200 import tp_dist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


S, H = 24, 16


def _partial_of(rank):
    g = torch.Generator().manual_seed(100 + rank)
    return torch.randn(S, H, generator=g)


def _x():
    return torch.randn(S, H, generator=torch.Generator().manual_seed(7))


def _worker(rank, world, port, mode, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    calls = []

    def partial(X, P, stream):
        P.copy_(_partial_of(rank))

    def reduce_ln(rows, parts, X_rows, Y_outs, stream):
        calls.append((rows, X_rows.clone()))
        z = X_rows[:rows] + sum(p[:rows] for p in parts)
        for y in Y_outs:
            y[:rows].copy_(z)

    sub = tp_dist.TPSublayer(partial, S, H, torch.float32, torch.float32, mode=mode, reduce_ln=reduce_ln)
    X = _x()
    Y = torch.full((S, H), float("nan"))
    sub.forward(X, Y)
    out[rank] = (Y, calls)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("mode", ["allreduce", "rs_ag"])  # the collective modes (peer mode: below)
def test_gloo_ranks_reduce_every_partial(world, mode):
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, mode, out), nprocs=world, join=True)
    X = _x()
    want = X + sum(_partial_of(r) for r in range(world))
    for r in range(world):
        Y, calls = out[r]
        torch.testing.assert_close(Y, want, rtol=1e-6, atol=1e-6)
        assert len(calls) == 1
        rows, X_rows = calls[0]
        if mode == "allreduce":
            assert rows == S and torch.equal(X_rows, X)
        else:
            r0, n = tp_dist.row_split(S, world, r)
            assert rows == n == S // world and torch.equal(X_rows, X[r0:r0 + n])


def test_row_split():
    assert tp_dist.row_split(2048, 4, 0) == (0, 512)
    assert tp_dist.row_split(2048, 4, 3) == (1536, 512)
    assert [tp_dist.row_split(12, 3, r) for r in range(3)] == [(0, 4), (4, 4), (8, 4)]
    with pytest.raises(ValueError):
        tp_dist.row_split(10, 4, 0)
    with pytest.raises(ValueError):
        tp_dist.row_split(8, 2, 2)


def test_single_rank_without_a_process_group():
    # world 1: no collective; both modes reduce the rank's own partial
    for mode in ("allreduce", "rs_ag"):
        def partial(X, P, stream):
            P.fill_(2.0)

        def reduce_ln(rows, parts, X_rows, Y_outs, stream):
            for y in Y_outs:
                y[:rows].copy_(X_rows[:rows] + parts[0][:rows])
        sub = tp_dist.TPSublayer(partial, 8, 4, torch.float32, torch.float32, mode=mode, reduce_ln=reduce_ln,
                                 world=1, rank=0)
        Y = sub.forward(torch.ones(8, 4), torch.zeros(8, 4))
        assert torch.equal(Y, torch.full((8, 4), 3.0))


class _FakePeerOps:
    """Stands in for CUDA IPC and the device barrier: handles are names,
    imports are made-up addresses, calls are recorded."""

    def __init__(self):
        self.calls = []

    def export(self, t):
        return ("handle", t.data_ptr())

    def import_(self, handle):
        return 10_000_000 + handle[1] % 1_000_003

    def close(self, addr):
        self.calls.append(("close", addr))

    def barrier(self, nranks, rank, flag_addrs, epoch, stream):
        self.calls.append(("barrier", nranks, rank, tuple(flag_addrs), epoch))


def test_peer_mode_bookkeeping():
    """Rank 1 of 2: the fused reduction reads rows [S/2, S) of both ranks'
    partials and writes them into both ranks' outputs, between two barriers
    with growing epochs; the imports are closed on close()."""
    S, H, world, rank = 8, 4, 2, 1
    ops = _FakePeerOps()
    theirs = {}

    def exchange(mine):
        other = tuple(("handle", 1000 + 64 * i) for i in range(3))  # rank 0's P, Ybuf, flags
        theirs["imports"] = [ops.import_(h) for h in other]
        return [other, mine]

    seen = []

    def partial(X, P, stream):
        P.fill_(1.0)

    def reduce_ln(rows, parts, X_rows, Y_outs, stream):
        seen.append((rows, list(parts), X_rows.clone(), list(Y_outs)))

    sub = tp_dist.TPSublayer(partial, S, H, torch.float32, torch.bfloat16, mode="peer", reduce_ln=reduce_ln,
                             world=world, rank=rank, peer_ops=ops, exchange=exchange)
    X = torch.arange(S * H, dtype=torch.float32).view(S, H)
    Y = torch.empty(S, H, dtype=torch.bfloat16)
    sub.Ybuf.fill_(3.0)
    sub.forward(X, Y)
    r0 = S // 2
    P0, Y0, F0 = theirs["imports"]
    assert sub.P_addr == [P0, sub.P.data_ptr()] and sub.Y_addr == [Y0, sub.Ybuf.data_ptr()]
    assert sub.F_addr == [F0, sub.flags.data_ptr()]
    (rows, parts, X_rows, outs), = seen
    assert rows == S // 2 and torch.equal(X_rows, X[r0:])
    assert parts == [P0 + r0 * H * 4, sub.P.data_ptr() + r0 * H * 4]
    assert outs == [Y0 + r0 * H * 2, sub.Ybuf.data_ptr() + r0 * H * 2]
    barriers = [c for c in ops.calls if c[0] == "barrier"]
    assert [b[4] for b in barriers] == [1, 2] and all(b[1:4] == (2, 1, tuple(sub.F_addr)) for b in barriers)
    assert torch.equal(Y, torch.full((S, H), 3.0, dtype=torch.bfloat16))  # copied from the shared output buffer
    sub.forward(X, Y)
    assert [c[4] for c in ops.calls if c[0] == "barrier"] == [1, 2, 3, 4]
    sub.close()
    assert sorted(c[1] for c in ops.calls if c[0] == "close") == sorted([P0, Y0, F0])
