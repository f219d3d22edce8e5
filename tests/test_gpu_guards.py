"""Out-of-bounds writes: every output (and workspace) buffer sits inside a
larger allocation whose guard regions before and after it are filled with a
byte pattern; after the call the guards must be unchanged.  Ragged shapes put
partial tiles at every edge the kernels clip (rows past M, columns past a
shard or the output width), in every GEMM tile shape (narrow 128-column
tiles, the cost model's choice, wide tiles)."""
from __future__ import annotations

import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import synth

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side
PATTERN = 0xA5


class Guarded:
    """A tensor view of `shape`/`dtype` inside a pattern-filled allocation."""

    def __init__(self, shape, dtype):
        n = 1
        for x in shape:
            n *= x
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        self.nbytes = nbytes
        self.raw = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(*shape) if nbytes else \
            torch.empty(shape, dtype=dtype, device="cuda")

    def intact(self) -> bool:
        g = torch.cat([self.raw[:GUARD], self.raw[GUARD + self.nbytes:]])
        return bool((g == PATTERN).all())


def _cuda(ts):
    return [x.cuda() for x in ts]


@pytest.mark.parametrize("tile_n", [0, 128, 480])
@pytest.mark.parametrize("S,H,F,t", [(200, 264, 1200, 3), (129, 1000, 2016, 2), (72, 72, 144, 1)])
def test_mlp_forward_and_training_writes_stay_in_bounds(cuda_device, tile_n, S, H, F, t):
    inp = synth.gen_mlp(S, H, F, seed=S)
    X = inp.X.cuda()
    As, Bs = _cuda(synth.split_columns(inp.A, t)), _cuda(synth.split_rows(inp.B, t))
    Y = Guarded((S, H), torch.bfloat16)
    ws = Guarded((L.mlp_workspace_bytes(S, H, F, t, X.dtype),), torch.uint8)
    state = Guarded((L.mlp_train_state_bytes(S, H, F, t),), torch.uint8)
    bws = Guarded((L.mlp_backward_workspace_bytes(S, H, F, t),), torch.uint8)
    dX = Guarded((S, H), torch.bfloat16)
    dA = [Guarded((H, F // t), torch.float32) for _ in range(t)]
    dB = [Guarded((F // t, H), torch.float32) for _ in range(t)]
    dg, db = Guarded((H,), torch.float32), Guarded((H,), torch.float32)
    dY, g, _ = synth.gen_upstream(S, H, seed=1)
    try:
        L.set_gemm_tile_n(tile_n)
        L.mlp_forward(X, As, Bs, Y.t, ws.t)
        L.mlp_forward_train(X, As, Bs, Y.t, state.t, gamma=g.cuda())
        L.mlp_backward(X, As, Bs, state.t, dY.cuda(), dX.t, [d.t for d in dA], [d.t for d in dB], bws.t,
                       gamma=g.cuda(), dgamma=dg.t, dbeta=db.t)
        torch.cuda.synchronize()
    finally:
        L.set_gemm_tile_n(0)
    assert L.device_error() == 0
    for name, buf in [("Y", Y), ("workspace", ws), ("state", state), ("backward workspace", bws), ("dX", dX),
                      ("dgamma", dg), ("dbeta", db)] + [(f"dA{i}", d) for i, d in enumerate(dA)] + \
            [(f"dB{i}", d) for i, d in enumerate(dB)]:
        assert buf.intact(), name


@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_linears_write_stay_in_bounds(cuda_device, out):
    inp = synth.gen_linear(300, 2 * 392, 2 * 1104, seed=3)
    X = inp.X.cuda()
    for fn, split in ((L.linear_column_forward, synth.split_columns), (L.linear_row_forward, synth.split_rows)):
        Y = Guarded((300, 2 * 1104), out)
        fn(X, _cuda(split(inp.W, 2)), Y.t)
        torch.cuda.synchronize()
        assert Y.intact(), fn.__name__


def test_attention_writes_stay_in_bounds(cuda_device):
    S, nh, d, t = 384, 4, 128, 2
    inp = synth.gen_attn(S, nh * d, seed=4)
    X = inp.X.cuda()
    Y = Guarded((S, nh * d), torch.bfloat16)
    ws = Guarded((L.attn_workspace_bytes(S, nh * d, nh, d, t),), torch.uint8)
    L.attn_forward(X, _cuda(synth.split_qkv_by_head(inp.Wqkv, nh, d, t)),
                   _cuda(synth.split_rows_by_head(inp.Wo, nh, d, t)), nh, d, Y.t, ws.t)
    torch.cuda.synchronize()
    assert Y.intact() and ws.intact()


@pytest.mark.parametrize("tile_n", [0, 128])
def test_attention_training_writes_stay_in_bounds(cuda_device, tile_n):
    """10 heads: a group of 8 and a group of 2 through the head-grouped GEMMs
    (the second group writes only part of the P / dS workspace), 384 rows (a
    partial 256-row tile)."""
    S, nh, d, t = 384, 10, 128, 2
    H = nh * d
    inp = synth.gen_attn(S, H, seed=5)
    dY, g, b = synth.gen_upstream(S, H, seed=6)
    X = inp.X.cuda()
    Wq = _cuda(synth.split_qkv_by_head(inp.Wqkv, nh, d, t))
    Wo = _cuda(synth.split_rows_by_head(inp.Wo, nh, d, t))
    Y = Guarded((S, H), torch.bfloat16)
    state = Guarded((L.attn_train_state_bytes(S, H, nh, d, t),), torch.uint8)
    bws = Guarded((L.attn_backward_workspace_bytes(S, H, nh, d, t),), torch.uint8)
    dX = Guarded((S, H), torch.bfloat16)
    dWq = [Guarded(tuple(w.shape), torch.float32) for w in Wq]
    dWo = [Guarded(tuple(w.shape), torch.float32) for w in Wo]
    dg, db = Guarded((H,), torch.float32), Guarded((H,), torch.float32)
    try:
        L.set_gemm_tile_n(tile_n)
        L.attn_forward_train(X, Wq, Wo, nh, d, Y.t, state.t, gamma=g.cuda(), beta=b.cuda())
        L.attn_backward(X, Wq, Wo, nh, d, state.t, dY.cuda(), dX.t, [w.t for w in dWq], [w.t for w in dWo], bws.t,
                        gamma=g.cuda(), dgamma=dg.t, dbeta=db.t)
        torch.cuda.synchronize()
    finally:
        L.set_gemm_tile_n(0)
    assert L.device_error() == 0
    for name, buf in [("Y", Y), ("state", state), ("backward workspace", bws), ("dX", dX), ("dgamma", dg),
                      ("dbeta", db)] + [(f"dWqkv{i}", w) for i, w in enumerate(dWq)] + \
            [(f"dWo{i}", w) for i, w in enumerate(dWo)]:
        assert buf.intact(), name


@pytest.mark.parametrize("S,H,F,t", [(77, 136, 312, 3), (128, 256, 1024, 2), (33, 40, 1040, 2)])
def test_mlp_f32_writes_stay_in_bounds(cuda_device, S, H, F, t):
    """The f32 CUDA-core path: ragged 32 x 32 tiles, and the row-split GEMM's
    K range cut over several f32 slots."""
    inp = synth.gen_mlp(S, H, F, seed=S + 1, dtype=torch.float32)
    X = inp.X.cuda()
    Y = Guarded((S, H), torch.float32)
    ws = Guarded((L.mlp_workspace_bytes(S, H, F, t, torch.float32),), torch.uint8)
    L.mlp_forward(X, _cuda(synth.split_columns(inp.A, t)), _cuda(synth.split_rows(inp.B, t)), Y.t, ws.t)
    torch.cuda.synchronize()
    assert Y.intact() and ws.intact()


def test_tp_partials_and_multi_output_reduce_stay_in_bounds(cuda_device):
    """Per-rank partial sums and the reduce + LayerNorm over pointer lists
    (row slices written into every output copy)."""
    S, H, F, N = 200, 264, 1200, 3
    inp = synth.gen_mlp(S, H, F, seed=9)
    X = inp.X.cuda()
    A, B = _cuda(synth.split_columns(inp.A, N)), _cuda(synth.split_rows(inp.B, N))
    parts, wss = [], []
    for r in range(N):
        P = Guarded((S, H), torch.float32)
        ws = Guarded((L.mlp_partial_workspace_bytes(S, H, F // N, 1),), torch.uint8)
        L.mlp_partial_forward(X, A[r:r + 1], B[r:r + 1], P.t, ws.t)
        parts.append(P)
        wss.append(ws)
    Ys = [Guarded((S, H), torch.bfloat16) for _ in range(N)]
    S_ = S - S % N
    for r in range(N):
        r0, n = r * (S_ // N), S_ // N
        L.reduce_residual_layernorm_multi(n, H, [p.t[r0:] for p in parts], X[r0:], [y.t[r0:] for y in Ys],
                                          torch.bfloat16, torch.bfloat16)
    torch.cuda.synchronize()
    assert all(b.intact() for b in parts + wss + Ys)
