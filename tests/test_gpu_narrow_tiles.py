"""GPU parity of the narrow-tile GEMM (128-column tiles; with an N-major B the
pair runs one N = 128 MMA, each CTA holding 64 B columns).  The cost model
picks narrow tiles for shards of at most 128 columns (the attention backward's
dV, dQ and dK GEMMs, whose N is the head dimension); here the tuning override
forces them on ragged shapes of every sublayer: column and row shard modes,
single CTAs (fewer than 129 rows) and CTA pairs, f32 and bf16 output, both
weight layouts (a K-major B keeps its 256-column MMA), a last tile that only
the first CTA of the pair loads, and the training step.  Same error metric and
bars as the other GPU parity tests.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import synth
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


def rel_err(got, ref) -> float:
    got = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / np.abs(ref).max())


@pytest.fixture
def narrow(cuda_device):
    L.set_gemm_tile_n(128)
    yield 128
    L.set_gemm_tile_n(0)


def _shards(ts, out_in):
    return [(x.t().contiguous() if out_in else x).cuda() for x in ts]


@pytest.mark.parametrize("out_in", [False, True])
@pytest.mark.parametrize("S,H,F,t", [
    (256, 512, 2048, 2),
    (300, 264, 1200, 3),     # H = 264: the row GEMM's last tile has 8 columns (second CTA loads no B)
    (520, 1000, 2016, 2),
    (100, 384, 1024, 2),     # 100 rows: single-CTA tiles
])
def test_mlp_narrow(narrow, out_in, S, H, F, t):
    inp = synth.gen_mlp(S, H, F, seed=S + H + t + 5, dtype=torch.bfloat16)
    X = inp.X.cuda()
    As = _shards(synth.split_columns(inp.A, t), out_in)
    Bs = _shards(synth.split_rows(inp.B, t), out_in)
    Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.mlp_workspace_bytes(S, H, F, t, X.dtype), dtype=torch.uint8, device="cuda")
    L.mlp_forward(X, As, Bs, Y, ws, layout="out_in" if out_in else "in_out")
    torch.cuda.synchronize()
    assert L.device_error() == 0
    assert rel_err(Y, O.mlp_block(inp.X, inp.A, inp.B)) <= TOL_BF16


@pytest.mark.parametrize("out_in", [False, True])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_linears_narrow(narrow, out_in, out):
    inp = synth.gen_linear(700, 2 * 392, 2 * 1104, seed=17)
    X = inp.X.cuda()
    layout = "out_in" if out_in else "in_out"
    Y = torch.empty(700, inp.W.shape[1], dtype=out, device="cuda")
    L.linear_column_forward(X, _shards(synth.split_columns(inp.W, 2), out_in), Y, act="gelu_tanh", layout=layout)
    torch.cuda.synchronize()
    assert rel_err(Y, O.linear_column(inp.X, inp.W, act="gelu_tanh")) <= TOL_BF16
    L.linear_row_forward(X, _shards(synth.split_rows(inp.W, 2), out_in), Y, layout=layout)
    torch.cuda.synchronize()
    assert rel_err(Y, O.linear_row(inp.X, inp.W)) <= TOL_BF16
    assert L.device_error() == 0


def test_attention_narrow(narrow):
    S, nh, d, t = 384, 6, 128, 2
    inp = synth.gen_attn(S, nh * d, seed=19)
    X = inp.X.cuda()
    H = nh * d
    Wq = [w.cuda() for w in synth.split_qkv_by_head(inp.Wqkv, nh, d, t)]
    Wo = [w.cuda() for w in synth.split_rows_by_head(inp.Wo, nh, d, t)]
    Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.attn_workspace_bytes(S, H, nh, d, t), dtype=torch.uint8, device="cuda")
    L.attn_forward(X, Wq, Wo, nh, d, Y, ws)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    assert rel_err(Y, O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d)) <= TOL_BF16


def test_mlp_training_step_narrow(narrow):
    """Every GEMM of the MLP training step (epilogue modes, M-major A, the
    M-split weight gradients) through 128-column tiles."""
    S, H, F, t = 300, 264, 1200, 3
    inp = synth.gen_mlp(S, H, F, seed=23, dtype=torch.bfloat16)
    dY, g, b = synth.gen_upstream(S, H, seed=24)
    X = inp.X.cuda()
    As = [a.cuda() for a in synth.split_columns(inp.A, t)]
    Bs = [x.cuda() for x in synth.split_rows(inp.B, t)]
    Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    state = torch.empty(L.mlp_train_state_bytes(S, H, F, t), dtype=torch.uint8, device="cuda")
    ws = torch.empty(L.mlp_backward_workspace_bytes(S, H, F, t), dtype=torch.uint8, device="cuda")
    gd, bd = g.cuda(), b.cuda()
    L.mlp_forward_train(X, As, Bs, Y, state, gamma=gd, beta=bd)
    dX = torch.empty_like(X)
    dA = [torch.empty(H, F // t, device="cuda") for _ in range(t)]
    dB = [torch.empty(F // t, H, device="cuda") for _ in range(t)]
    dg = torch.empty(H, device="cuda")
    db = torch.empty(H, device="cuda")
    L.mlp_backward(X, As, Bs, state, dY.cuda(), dX, dA, dB, ws, gamma=gd, dgamma=dg, dbeta=db)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    ref = O.mlp_block_backward(inp.X, inp.A, inp.B, dY, g)
    got = {"dX": dX, "dA": torch.cat(dA, 1), "dB": torch.cat(dB, 0), "dgamma": dg, "dbeta": db}
    errs = {k: rel_err(got[k], ref[k]) for k in got}
    assert all(e <= TOL_BF16 for e in errs.values()), errs


def test_attention_backward_narrow(narrow):
    """The attention training step with every GEMM on 128-column tiles (the
    softmax epilogues included)."""
    S, nh, d, t = 384, 4, 128, 2
    H = nh * d
    inp = synth.gen_attn(S, H, seed=29)
    dY, g, b = synth.gen_upstream(S, H, seed=30)
    X = inp.X.cuda()
    Wq = [w.cuda() for w in synth.split_qkv_by_head(inp.Wqkv, nh, d, t)]
    Wo = [w.cuda() for w in synth.split_rows_by_head(inp.Wo, nh, d, t)]
    Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    state = torch.empty(L.attn_train_state_bytes(S, H, nh, d, t), dtype=torch.uint8, device="cuda")
    L.attn_forward_train(X, Wq, Wo, nh, d, Y, state, gamma=g.cuda(), beta=b.cuda())
    dX = torch.empty_like(Y)
    dWq = [torch.empty(*w.shape, dtype=torch.float32, device="cuda") for w in Wq]
    dWo = [torch.empty(*w.shape, dtype=torch.float32, device="cuda") for w in Wo]
    dg = torch.empty(H, device="cuda")
    db = torch.empty(H, device="cuda")
    ws = torch.empty(L.attn_backward_workspace_bytes(S, H, nh, d, t), dtype=torch.uint8, device="cuda")
    L.attn_backward(X, Wq, Wo, nh, d, state, dY.cuda(), dX, dWq, dWo, ws, gamma=g.cuda(), dgamma=dg, dbeta=db)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    ref = O.attention_sublayer_backward(inp.X, inp.Wqkv, inp.Wo, nh, d, dY, g, b)
    ref_q = synth.split_qkv_by_head(torch.from_numpy(ref["dWqkv"]), nh, d, t)
    ref_o = synth.split_rows_by_head(torch.from_numpy(ref["dWo"]), nh, d, t)
    errs = {"dX": rel_err(dX, ref["dX"]), "dgamma": rel_err(dg, ref["dgamma"]), "dbeta": rel_err(db, ref["dbeta"])}
    for s in range(t):
        errs[f"dWqkv{s}"] = rel_err(dWq[s], ref_q[s].numpy())
        errs[f"dWo{s}"] = rel_err(dWo[s], ref_o[s].numpy())
    assert all(e <= TOL_BF16 for e in errs.values()), errs
