"""The N > 1 host path of bench.py on CPU: two gloo ranks agree on the max of
their timings and on the whole-job (weak-scaling) throughput."""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    mine = [10.0 + rank * 5.0, 3.0 - rank]          # rank 1 is slower on the first
    got = bench.max_over_ranks(mine, world)
    out[rank] = got + [bench.whole_job_tflops(1_000_000_000_000, 10, world, got[0])]
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_max_and_weak_scaling_value():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1]
    ms_max, e2e_max, value = out[0]
    assert ms_max == 15.0 and e2e_max == 3.0
    # 2 ranks x 10 steps x 1e12 FLOP in 15 ms
    assert value == pytest.approx(2 * 10 * 1e12 / 15e-3 / 1e12)


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]
