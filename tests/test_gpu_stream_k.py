"""Stream-K scheduling of the tensor-core GEMM (tp_set_gemm_stream_k): whole
waves of tiles, then the remainder tiles split along K between the pairs that
run their heads (and finish them, after a bounded wait for the tails' f32
partials) and the spare pairs that run their tails.

Forced on (1) for small ragged shapes, in every tile shape (the cost model's
width, 256, wide and narrow tiles), over as many pairs as the sublayer's spare
partial-sum slots hold partial blocks for (whole waves, then the remainder
tiles split between head and tail pieces); checked against the fp64 oracle,
against the whole-tile schedule (-1), and for run-to-run bitwise repeatability.
The full-size workloads take stream-K by default (the cost model), so the
full-size parity tests cover it at the sizes bench.py times."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import synth
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu

TOL = 2e-2


def rel_err(Y, ref):
    got = Y.double().cpu().numpy()
    return float(np.abs(got - ref).max() / np.abs(ref).max())


@pytest.fixture
def sk_mode():
    yield L.set_gemm_stream_k
    L.set_gemm_stream_k(0)
    L.set_gemm_tile_n(0)


def _mlp(inp, t, Y, ws, gamma=None, beta=None):
    L.mlp_forward(inp.Xd, inp.Ad, inp.Bd, Y, ws, gamma=gamma, beta=beta)
    torch.cuda.synchronize()
    assert L.device_error() == 0


@pytest.mark.parametrize("tile_n", [0, 256, 384, 512, 128])
@pytest.mark.parametrize("S,H,F,t", [(600, 520, 2240, 2), (384, 1024, 4096, 4), (300, 640, 1200, 3),
                                     (1000, 768, 3072, 8)])
def test_mlp_stream_k_matches_oracle_and_whole_tiles(cuda_device, sk_mode, tile_n, S, H, F, t):
    inp = synth.gen_mlp(S, H, F, seed=S + t)
    inp.Xd = inp.X.cuda()
    inp.Ad = [a.cuda() for a in synth.split_columns(inp.A, t)]
    inp.Bd = [b.cuda() for b in synth.split_rows(inp.B, t)]
    g = torch.Generator().manual_seed(t)
    gamma, beta = 1.0 + 0.25 * torch.randn(H, generator=g), 0.25 * torch.randn(H, generator=g)
    ws = torch.empty(L.mlp_workspace_bytes(S, H, F, t, torch.bfloat16), dtype=torch.uint8, device="cuda")
    L.set_gemm_tile_n(tile_n)
    # forced on, at least one of the two GEMMs has remainder tiles to split
    # (the other may divide evenly over the pairs the spare slots allow)
    area = 3 * S * H * 4
    sk_mode(1)
    plans = [L.gemm_plan_sk(S, t, row, sk_, sn, f32, max_splits=4 if f32 else 1, sk_area_bytes=area)
             for row, sk_, sn, f32 in ((0, H, F // t, 0), (1, F // t, H, 1))]
    assert any(pl[2] == 1 and pl[3] >= 2 for pl in plans), plans
    Ys = []
    for _ in range(2):
        Y = torch.full((S, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        _mlp(inp, t, Y, ws, gamma.cuda(), beta.cuda())
        Ys.append(Y)
    assert torch.equal(Ys[0], Ys[1]), "stream-K results differ between runs"
    ref = O.mlp_block(inp.X, inp.A, inp.B, gamma=gamma, beta=beta)
    assert rel_err(Ys[0], ref) <= TOL
    sk_mode(0)
    Yw = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    _mlp(inp, t, Yw, ws, gamma.cuda(), beta.cuda())
    assert rel_err(Yw, ref) <= TOL
    # the two schedules sum the same products in different orders: close, not equal
    assert rel_err(Ys[0], Yw.double().cpu().numpy()) <= TOL


@pytest.mark.parametrize("tile_n", [0, 512])
def test_attention_stream_k(cuda_device, sk_mode, tile_n):
    S, nh, d, t = 512, 8, 128, 4
    H = nh * d
    inp = synth.gen_attn(S, H, seed=11)
    X = inp.X.cuda()
    Wq = [w.cuda() for w in synth.split_qkv_by_head(inp.Wqkv, nh, d, t)]
    Wo = [w.cuda() for w in synth.split_rows_by_head(inp.Wo, nh, d, t)]
    ws = torch.empty(L.attn_workspace_bytes(S, H, nh, d, t), dtype=torch.uint8, device="cuda")
    L.set_gemm_tile_n(tile_n)
    sk_mode(1)
    Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    L.attn_forward(X, Wq, Wo, nh, d, Y, ws)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    assert rel_err(Y, O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d)) <= TOL


def test_stream_k_writes_stay_inside_the_workspace(cuda_device, sk_mode):
    """The partial blocks and flags live in the spare slots of the caller's
    workspace: guard regions around Y and the workspace stay untouched."""
    S, H, F, t = 600, 520, 2240, 2
    inp = synth.gen_mlp(S, H, F, seed=3)
    guard = 4096
    ws_bytes = L.mlp_workspace_bytes(S, H, F, t, torch.bfloat16)
    raw_ws = torch.full((guard + ws_bytes + guard,), 0xA5, dtype=torch.uint8, device="cuda")
    raw_y = torch.full((guard + S * H * 2 + guard,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = raw_ws[guard:guard + ws_bytes]
    Y = raw_y[guard:guard + S * H * 2].view(torch.bfloat16).view(S, H)
    sk_mode(1)
    L.mlp_forward(inp.X.cuda(), [a.cuda() for a in synth.split_columns(inp.A, t)],
                  [b.cuda() for b in synth.split_rows(inp.B, t)], Y, ws)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    for raw, n in ((raw_ws, ws_bytes), (raw_y, S * H * 2)):
        assert bool((raw[:guard] == 0xA5).all()) and bool((raw[guard + n:] == 0xA5).all())
    assert rel_err(Y, O.mlp_block(inp.X, inp.A, inp.B)) <= TOL
