"""GPU parity of the wide-tile GEMM (tiles of up to 512 columns, two MMAs per K
step filling TMEM).  The library's cost model picks wide tiles only for some
full-size shapes; here the tuning override forces them on small ragged shapes
so that both weight layouts, both shard modes, both output types, ragged last
tiles (a tile with no second MMA, a second MMA that only one CTA of the pair
loads) and the attention sublayer run through them.  Same error metric and bars
as the other GPU parity tests.
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
def tile_n(request, cuda_device):
    L.set_gemm_tile_n(request.param)
    yield request.param
    L.set_gemm_tile_n(0)


def _shards(ts, out_in):
    return [(x.t().contiguous() if out_in else x).cuda() for x in ts]


@pytest.mark.parametrize("tile_n", [288, 480, 512], indirect=True)
@pytest.mark.parametrize("out_in", [False, True])
@pytest.mark.parametrize("S,H,F,t", [
    (256, 512, 2048, 2),
    (300, 264, 1200, 3),     # ragged rows, ragged K, shard width 400, H=264: last tile 264-w... < 256
    (520, 1000, 2016, 2),    # H = 1000: second MMA of the last tile loaded by one CTA only
])
def test_mlp_wide(tile_n, out_in, S, H, F, t):
    inp = synth.gen_mlp(S, H, F, seed=S + H + t, dtype=torch.bfloat16)
    X = inp.X.cuda()
    As = _shards(synth.split_columns(inp.A, t), out_in)
    Bs = _shards(synth.split_rows(inp.B, t), out_in)
    Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.mlp_workspace_bytes(S, H, F, t, X.dtype), dtype=torch.uint8, device="cuda")
    L.mlp_forward(X, As, Bs, Y, ws, layout="out_in" if out_in else "in_out")
    torch.cuda.synchronize()
    assert L.device_error() == 0
    assert rel_err(Y, O.mlp_block(inp.X, inp.A, inp.B)) <= TOL_BF16


@pytest.mark.parametrize("tile_n", [384, 480], indirect=True)
@pytest.mark.parametrize("out_in", [False, True])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_linears_wide(tile_n, out_in, out):
    inp = synth.gen_linear(700, 2 * 392, 2 * 1104, seed=tile_n)
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


@pytest.mark.parametrize("tile_n", [480], indirect=True)
def test_attention_wide(tile_n):
    S, nh, d, t = 384, 6, 128, 2
    inp = synth.gen_attn(S, nh * d, seed=9)
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


def test_wide_and_narrow_agree(cuda_device):
    """Same operands through 256-column tiles and wide tiles: both within the
    bar of the oracle and of each other."""
    inp = synth.gen_mlp(512, 1024, 4096, seed=21, dtype=torch.bfloat16)
    X = inp.X.cuda()
    As = _shards(synth.split_columns(inp.A, 4), False)
    Bs = _shards(synth.split_rows(inp.B, 4), False)
    ws = torch.empty(L.mlp_workspace_bytes(512, 1024, 4096, 4, X.dtype), dtype=torch.uint8, device="cuda")
    ys = {}
    try:
        for w in (256, 480):
            L.set_gemm_tile_n(w)
            Y = torch.empty(512, 1024, dtype=torch.bfloat16, device="cuda")
            L.mlp_forward(X, As, Bs, Y, ws)
            torch.cuda.synchronize()
            ys[w] = Y
    finally:
        L.set_gemm_tile_n(0)
    ref = O.mlp_block(inp.X, inp.A, inp.B)
    for y in ys.values():
        assert rel_err(y, ref) <= TOL_BF16
    assert rel_err(ys[480], ys[256].double().cpu().numpy()) <= TOL_BF16
