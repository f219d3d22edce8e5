"""The fused multi-GPU reduction's plumbing, checked on one GPU.

* CUDA IPC between two processes on the same GPU: rank 0 exports its partial
  sum buffer (a piece of a larger allocation, so the handle's offset
  matters); rank 1 maps it and runs tp_reduce_residual_layernorm_multi with
  one partial read through the mapping and one of its own, writing both its
  own output and, through a second mapping, rank 0's output buffer.  No
  kernel waits on another: rank 0 only waits on the host (a gloo barrier)
  until rank 1 is done, then checks what landed in its buffer.
* The device-side barrier with the other rank's arrival already in this
  rank's flags (set by a copy before the launch): the kernel must store its
  own arrival into the other rank's array and return without timing out; and
  the single-rank barrier.  Nothing waits on a second process's kernel."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from megatron_tensor_transformer_gelu_b200 import _lib as L

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


S, H = 64, 256


def _data(seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(S, H, generator=g)


def _ipc_worker(rank, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2)
    torch.cuda.set_device(0)
    try:
        if rank == 0:
            # the partial sits 4 KiB into a larger buffer: the handle must carry the offset
            big = torch.zeros(S * H + 1024, dtype=torch.float32, device="cuda")
            P0 = big[1024:].view(S, H)
            P0.copy_(_data(1).cuda())
            Yb = torch.zeros(S * H + 512, dtype=torch.bfloat16, device="cuda")
            Y0 = Yb[512:].view(S, H)
            torch.cuda.synchronize()
            handles = [L.ipc_export(P0), L.ipc_export(Y0)]
            dist.broadcast_object_list([handles], src=0)
            dist.barrier()  # rank 1 has run its kernel and synchronised
            out[0] = Y0.float().cpu()
        else:
            box = [None]
            dist.broadcast_object_list(box, src=0)
            p0 = L.ipc_import(box[0][0])
            y0 = L.ipc_import(box[0][1])
            P1 = _data(2).cuda()
            X = _data(3).to(torch.bfloat16).cuda()
            Y1 = torch.zeros(S, H, dtype=torch.bfloat16, device="cuda")
            # rows [16, 48): a slice, as one rank's share of the rows
            r0, n = 16, 32
            L.reduce_residual_layernorm_multi(n, H, [p0 + r0 * H * 4, P1[r0:]], X[r0:], [Y1[r0:], y0 + r0 * H * 2],
                                              torch.bfloat16, torch.bfloat16)
            torch.cuda.synchronize()
            out[1] = (Y1.float().cpu(), L.device_error())
            L.ipc_close(p0)
            L.ipc_close(y0)
            dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ipc_partial_and_output_between_two_processes(cuda_device):
    from oracle import tp_oracle as O
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_ipc_worker, args=(port, out), nprocs=2, join=True, start_method="spawn")
    Y1, err = out[1]
    assert err == 0
    X = _data(3).to(torch.bfloat16).double().numpy()
    r0, n = 16, 32
    ref = O.layernorm(X[r0:r0 + n] + _data(1).double().numpy()[r0:r0 + n] + _data(2).double().numpy()[r0:r0 + n])
    got1 = Y1.double().numpy()
    assert np.abs(got1[r0:r0 + n] - ref).max() / np.abs(ref).max() <= 1e-2
    assert not got1[:r0].any() and not got1[r0 + n:].any()  # only the slice was written
    got0 = out[0].double().numpy()  # the same rows, stored through the mapping into rank 0's buffer
    np.testing.assert_array_equal(got0[r0:r0 + n], got1[r0:r0 + n])
    assert not got0[:r0].any() and not got0[r0 + n:].any()


def test_peer_barrier_with_the_other_arrival_already_present(cuda_device):
    mine = torch.zeros(2, dtype=torch.int64, device="cuda")
    theirs = torch.zeros(2, dtype=torch.int64, device="cuda")
    mine[1] = 1  # rank 1 has arrived at epoch 1
    torch.cuda.synchronize()
    L.peer_barrier(2, 0, [mine, theirs], 1)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    assert mine.tolist() == [1, 1] and theirs.tolist() == [1, 0]  # our arrival in both arrays' slot 0
    # a later epoch: arrivals are compared with >=, so a peer one barrier ahead also counts
    mine[1] = 3
    L.peer_barrier(2, 0, [mine, theirs], 2)
    torch.cuda.synchronize()
    assert L.device_error() == 0 and theirs.tolist() == [2, 0]


def test_peer_barrier_single_rank_and_bad_arguments(cuda_device):
    f = torch.zeros(1, dtype=torch.int64, device="cuda")
    for e in (1, 2, 3):
        L.peer_barrier(1, 0, [f], e)
    torch.cuda.synchronize()
    assert L.device_error() == 0 and f.item() == 3
    for args in ((0, 0, [f], 1), (1, 1, [f], 1), (1, 0, [f], 0), (9, 0, [f] * 9, 1)):
        with pytest.raises(L.TPError):
            L.peer_barrier(*args)
