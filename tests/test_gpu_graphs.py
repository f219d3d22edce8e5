"""CUDA-graph capture and replay of the sublayer calls.

The calls allocate nothing and never synchronise, so a call captured into a
CUDA graph replays the same launches.  Each case makes one direct call,
captures the same call on a side stream, replays the graph several times with
the output cleared in between, and compares every replay bit for bit with the
direct call (the kernels are deterministic: fixed reduction orders, plain
stores), and the direct call with the fp64 oracle.  The attention forward
runs with every unit's keys split in two and with the default split of the
last partial wave: the split's claim / ready flags carry one epoch for all
replays of a graph, so each replay must find them unclaimed.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import synth
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu

REPLAYS = 3


def rel_err(got, ref) -> float:
    got = got.detach().double().cpu().numpy()
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / np.abs(ref).max())


def replay_matches(call, outs):
    """Capture call(stream) once, replay it REPLAYS times, compare `outs` with
    their values after the direct call."""
    call(torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert L.device_error() == 0
    refs = [o.clone() for o in outs]
    side = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        call(side)
    for _ in range(REPLAYS):
        for o in outs:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert L.device_error() == 0
        for o, r in zip(outs, refs):
            assert torch.equal(o, r), "a replay differs from the direct call"
    del graph
    return refs


@pytest.mark.parametrize("dtype,S,H,F,t,tol", [(torch.bfloat16, 512, 1024, 4096, 2, 2e-2),
                                               (torch.float32, 128, 256, 1024, 2, 1e-4)])
def test_mlp_forward_replays(cuda_device, dtype, S, H, F, t, tol):
    inp = synth.gen_mlp(S, H, F, seed=7, dtype=dtype)
    X = inp.X.cuda()
    A = [a.cuda() for a in synth.split_columns(inp.A, t)]
    B = [b.cuda() for b in synth.split_rows(inp.B, t)]
    Y = torch.empty(S, H, dtype=dtype, device="cuda")
    ws = torch.empty(L.mlp_workspace_bytes(S, H, F, t, dtype), dtype=torch.uint8, device="cuda")
    (ref,) = replay_matches(lambda st: L.mlp_forward(X, A, B, Y, ws, stream=st), [Y])
    assert rel_err(ref, O.mlp_block(inp.X, inp.A, inp.B)) <= tol


@pytest.mark.parametrize("mode", [2, 1])
def test_attention_forward_replays_with_key_split(cuda_device, mode):
    S, nh, d, t = 640, 4, 128, 2
    H = nh * d
    inp = synth.gen_attn(S, H, seed=11)
    X = inp.X.cuda()
    Wq = [w.cuda() for w in synth.split_qkv_by_head(inp.Wqkv, nh, d, t)]
    Wo = [w.cuda() for w in synth.split_rows_by_head(inp.Wo, nh, d, t)]
    Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.attn_workspace_bytes(S, H, nh, d, t), dtype=torch.uint8, device="cuda")
    L.set_attn_kv_split(mode)
    try:
        (ref,) = replay_matches(lambda st: L.attn_forward(X, Wq, Wo, nh, d, Y, ws, stream=st), [Y])
    finally:
        L.set_attn_kv_split(1)
    assert rel_err(ref, O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d)) <= 2e-2


def test_mlp_training_step_replays(cuda_device):
    S, H, F, t = 256, 512, 2048, 2
    inp = synth.gen_mlp(S, H, F, seed=5)
    dY, gamma, _ = synth.gen_upstream(S, H, seed=6)
    X = inp.X.cuda()
    A = [a.cuda() for a in synth.split_columns(inp.A, t)]
    B = [b.cuda() for b in synth.split_rows(inp.B, t)]
    g = gamma.cuda()
    dYd = dY.cuda()
    Yf = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    dX = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    state = torch.empty(L.mlp_train_state_bytes(S, H, F, t), dtype=torch.uint8, device="cuda")
    ws = torch.empty(L.mlp_backward_workspace_bytes(S, H, F, t), dtype=torch.uint8, device="cuda")
    dA = [torch.empty(H, F // t, dtype=torch.float32, device="cuda") for _ in range(t)]
    dB = [torch.empty(F // t, H, dtype=torch.float32, device="cuda") for _ in range(t)]
    dg = torch.empty(H, dtype=torch.float32, device="cuda")
    db = torch.empty(H, dtype=torch.float32, device="cuda")

    def step(st):
        L.mlp_forward_train(X, A, B, Yf, state, gamma=g, stream=st)
        L.mlp_backward(X, A, B, state, dYd, dX, dA, dB, ws, gamma=g, dgamma=dg, dbeta=db, stream=st)

    refs = replay_matches(step, [Yf, dX, *dA, *dB, dg, db])
    want = O.mlp_block_backward(inp.X, inp.A, inp.B, dY, gamma)
    assert rel_err(refs[1], want["dX"]) <= 2e-2
