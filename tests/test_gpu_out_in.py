"""GPU parity for the nn.Linear weight layout ([out, in] shards, `x @ W.T`).

Weights stored [out, in] are the transposes of the [in, out] shards the
sublayer is written in (Megatron-LM paper, "Model Parallel Transformers",
section 3, with PyTorch's Linear convention); the kernels read them K-major
without a transpose pass.  Each case builds the [in, out] shards the other
parity tests use, passes their transposes, and compares with the fp64 oracle
on the untransposed weights.  Same error metric and bars as the other GPU
parity tests.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import synth
from megatron_tensor_transformer_gelu_b200.workloads import WORKLOADS
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
TOL_F32 = 1e-4


def rel_err(got, ref) -> float:
    got = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / np.abs(ref).max())


def _t(ts):
    return [t.t().contiguous().cuda() for t in ts]


def _d(ts):
    return [t.cuda() for t in ts]


def run_mlp(inp, t, layout, act="gelu_tanh"):
    X = inp.X.cuda()
    S, H = X.shape
    F = inp.A.shape[1]
    As = synth.split_columns(inp.A, t)
    Bs = synth.split_rows(inp.B, t)
    As, Bs = (_t(As), _t(Bs)) if layout == "out_in" else (_d(As), _d(Bs))
    Y = torch.empty(S, H, dtype=X.dtype, device="cuda")
    ws = torch.empty(max(1, L.mlp_workspace_bytes(S, H, F, t, X.dtype)), dtype=torch.uint8, device="cuda")
    L.mlp_forward(X, As, Bs, Y, ws, act=act, layout=layout)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    return Y


@pytest.mark.parametrize("S,H,F,t", [
    (256, 256, 1024, 2),
    (200, 264, 1200, 3),     # ragged rows, ragged K, shard width 400 (ragged N tile)
    (129, 512, 2048, 8),
    (1, 64, 64, 1),
])
def test_mlp_bf16_out_in(cuda_device, S, H, F, t):
    inp = synth.gen_mlp(S, H, F, seed=S + H, dtype=torch.bfloat16)
    Y = run_mlp(inp, t, "out_in")
    assert rel_err(Y, O.mlp_block(inp.X, inp.A, inp.B)) <= TOL_BF16
    Y0 = run_mlp(inp, t, "in_out")
    assert rel_err(Y, Y0.double().cpu().numpy()) <= 1e-2


def test_mlp_f32_out_in(cuda_device):
    inp = synth.gen_mlp(77, 136, 3 * 104, seed=3, dtype=torch.float32)
    Y = run_mlp(inp, 3, "out_in", act="gelu_erf")
    assert rel_err(Y, O.mlp_block(inp.X, inp.A, inp.B, act="gelu_erf")) <= TOL_F32


@pytest.mark.parametrize("S,nh,t", [(256, 4, 2), (384, 4, 4)])
def test_attention_out_in(cuda_device, S, nh, t):
    d = 128
    inp = synth.gen_attn(S, nh * d, seed=S + nh)
    X = inp.X.cuda()
    H = nh * d
    Wq = _t(synth.split_qkv_by_head(inp.Wqkv, nh, d, t))
    Wo = _t(synth.split_rows_by_head(inp.Wo, nh, d, t))
    Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.attn_workspace_bytes(S, H, nh, d, t), dtype=torch.uint8, device="cuda")
    L.attn_forward(X, Wq, Wo, nh, d, Y, ws, layout="out_in")
    torch.cuda.synchronize()
    assert L.device_error() == 0
    ref = O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d)
    assert rel_err(Y, ref) <= TOL_BF16


@pytest.mark.parametrize("t", [1, 2, 4])
def test_linears_bf16_out_in(cuda_device, t):
    inp = synth.gen_linear(300, 4 * 136, 8 * 3 * 40, seed=t)
    X = inp.X.cuda()
    Y = torch.empty(300, inp.W.shape[1], dtype=torch.float32, device="cuda")
    L.linear_column_forward(X, _t(synth.split_columns(inp.W, t)), Y, layout="out_in")
    torch.cuda.synchronize()
    assert rel_err(Y, O.linear_column(inp.X, inp.W)) <= TOL_BF16
    L.linear_row_forward(X, _t(synth.split_rows(inp.W, t)), Y, layout="out_in")
    torch.cuda.synchronize()
    assert rel_err(Y, O.linear_row(inp.X, inp.W)) <= TOL_BF16


def test_linears_f32_out_in(cuda_device):
    inp = synth.gen_linear(70, 96, 160, seed=1, dtype=torch.float32)
    X = inp.X.cuda()
    Y = torch.empty(70, 160, dtype=torch.float32, device="cuda")
    L.linear_column_forward(X, _t(synth.split_columns(inp.W, 2)), Y, act="relu", layout="out_in")
    torch.cuda.synchronize()
    assert rel_err(Y, O.linear_column(inp.X, inp.W, act="relu")) <= TOL_F32
    L.linear_row_forward(X, _t(synth.split_rows(inp.W, 4)), Y, layout="out_in")
    torch.cuda.synchronize()
    assert rel_err(Y, O.linear_row(inp.X, inp.W)) <= TOL_F32


@pytest.mark.slow
def test_mlp_s2048_h4096_f16384_out_in(cuda_device):
    w = WORKLOADS["mlp_s2048_h4096_f16384"]
    inp = synth.gen_mlp(w.S, w.H, w.F, seed=w.seed)
    Y = run_mlp(inp, 4, "out_in")
    rows = synth.row_sample(w.S, w.seed + 1)
    assert rel_err(Y[rows], O.mlp_block(inp.X, inp.A, inp.B, rows=rows)) <= TOL_BF16

