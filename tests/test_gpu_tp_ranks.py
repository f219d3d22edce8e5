"""The multi-GPU form of the sublayers, checked on one GPU.

Each rank's partial sum is computed in turn by the per-rank entry points
(tp_mlp_partial_forward / tp_attn_partial_forward) from that rank's shards;
the reduction is then run as the multi-GPU forms run it, over the ranks'
buffers held on this GPU (no kernel waits on another):
  * the AllReduce form: one tp_reduce_residual_layernorm_multi over all rows
    with every rank's partial;
  * the ReduceScatter -> LayerNorm on S/N rows -> AllGather form: one call per
    rank on its slice of the rows, reading every rank's partial and writing
    every rank's output buffer, as the peer-access form does across GPUs.
Both are compared with the fp64 oracle of the unsplit sublayer, and every
rank's output buffer must hold the same values."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import synth, tp_dist
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu

TOL_BF16, TOL_F32 = 2e-2, 1e-4


def rel_err(Y, ref):
    got = Y.double().cpu().numpy()
    return float(np.abs(got - ref).max() / np.abs(ref).max())


def _reduce_both_ways(parts, X, gamma, beta, out_dtype):
    """(Y of the AllReduce form, [each rank's Y] of the ReduceScatter/AllGather form)."""
    S, H = X.shape
    N = len(parts)
    Y = torch.full((S, H), float("nan"), dtype=out_dtype, device="cuda")
    L.reduce_residual_layernorm_multi(S, H, parts, X, [Y], X.dtype, out_dtype, gamma=gamma, beta=beta)
    Ys = [torch.full((S, H), float("nan"), dtype=out_dtype, device="cuda") for _ in range(N)]
    for r in range(N):
        r0, n = tp_dist.row_split(S, N, r)
        L.reduce_residual_layernorm_multi(n, H, [p[r0:] for p in parts], X[r0:], [y[r0:] for y in Ys], X.dtype,
                                          out_dtype, gamma=gamma, beta=beta)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    return Y, Ys


def _ln_params(H, seed):
    g = torch.Generator().manual_seed(seed)
    return 1.0 + 0.25 * torch.randn(H, generator=g), 0.25 * torch.randn(H, generator=g)


@pytest.mark.parametrize("S,H,F,N,per_rank", [(256, 512, 2048, 2, 1), (384, 256, 4096, 4, 1),
                                              (200, 512, 2048, 8, 1), (256, 384, 3072, 2, 3)])
def test_mlp_ranks_in_turn(cuda_device, S, H, F, N, per_rank):
    inp = synth.gen_mlp(S, H, F, seed=S + N)
    gamma, beta = _ln_params(H, N)
    X = inp.X.cuda()
    t = N * per_rank
    A = [a.cuda() for a in synth.split_columns(inp.A, t)]
    B = [b.cuda() for b in synth.split_rows(inp.B, t)]
    parts = []
    for r in range(N):
        mine = slice(r * per_rank, (r + 1) * per_rank)
        Fr = F // N
        ws = torch.empty(L.mlp_partial_workspace_bytes(S, H, Fr, per_rank), dtype=torch.uint8, device="cuda")
        P = torch.full((S, H), float("nan"), dtype=torch.float32, device="cuda")
        L.mlp_partial_forward(X, A[mine], B[mine], P, ws)
        parts.append(P)
    Y, Ys = _reduce_both_ways(parts, X, gamma.cuda(), beta.cuda(), torch.bfloat16)
    ref = O.mlp_block(inp.X, inp.A, inp.B, gamma=gamma, beta=beta)
    assert rel_err(Y, ref) <= TOL_BF16
    for y in Ys:
        assert torch.equal(y, Y)  # same kernel, same partials in the same order: the same bits
    # the one-GPU sublayer (all shards on this GPU) agrees within the tolerance too
    Y1 = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    L.mlp_forward(X, A, B, Y1, torch.empty(L.mlp_workspace_bytes(S, H, F, t, torch.bfloat16), dtype=torch.uint8,
                                            device="cuda"), gamma=gamma.cuda(), beta=beta.cuda())
    torch.cuda.synchronize()
    assert rel_err(Y1, ref) <= TOL_BF16


def test_mlp_ranks_in_turn_f32(cuda_device):
    S, H, F, N = 128, 256, 1024, 2
    inp = synth.gen_mlp(S, H, F, seed=0, dtype=torch.float32)
    X = inp.X.cuda()
    A = [a.cuda() for a in synth.split_columns(inp.A, N)]
    B = [b.cuda() for b in synth.split_rows(inp.B, N)]
    parts = []
    for r in range(N):
        ws = torch.empty(L.mlp_partial_workspace_bytes(S, H, F // N, 1, torch.float32), dtype=torch.uint8,
                         device="cuda")
        P = torch.empty(S, H, dtype=torch.float32, device="cuda")
        L.mlp_partial_forward(X, A[r:r + 1], B[r:r + 1], P, ws)
        parts.append(P)
    Y, Ys = _reduce_both_ways(parts, X, None, None, torch.float32)
    ref = O.mlp_block(inp.X, inp.A, inp.B)
    assert rel_err(Y, ref) <= TOL_F32
    assert all(torch.equal(y, Y) for y in Ys)


@pytest.mark.parametrize("S,nh,N", [(256, 4, 2), (256, 8, 4), (384, 8, 8)])
def test_attention_ranks_in_turn(cuda_device, S, nh, N):
    d = 128
    H = nh * d
    inp = synth.gen_attn(S, H, seed=S + nh)
    gamma, beta = _ln_params(H, nh)
    X = inp.X.cuda()
    Wq = [w.cuda() for w in synth.split_qkv_by_head(inp.Wqkv, nh, d, N)]
    Wo = [w.cuda() for w in synth.split_rows_by_head(inp.Wo, nh, d, N)]
    parts = []
    for r in range(N):
        nh_r = nh // N
        ws = torch.empty(L.attn_partial_workspace_bytes(S, H, nh_r, d, 1), dtype=torch.uint8, device="cuda")
        P = torch.full((S, H), float("nan"), dtype=torch.float32, device="cuda")
        L.attn_partial_forward(X, Wq[r:r + 1], Wo[r:r + 1], nh_r, d, P, ws)
        parts.append(P)
    Y, Ys = _reduce_both_ways(parts, X, gamma.cuda(), beta.cuda(), torch.bfloat16)
    ref = O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d, gamma=gamma, beta=beta)
    assert rel_err(Y, ref) <= TOL_BF16
    assert all(torch.equal(y, Y) for y in Ys)


def test_attention_rank_with_two_head_shards(cuda_device):
    # one rank holding 2 of the 4 head shards: its partial is the sum of both
    S, nh, d = 256, 8, 128
    H = nh * d
    inp = synth.gen_attn(S, H, seed=5)
    X = inp.X.cuda()
    Wq = [w.cuda() for w in synth.split_qkv_by_head(inp.Wqkv, nh, d, 4)]
    Wo = [w.cuda() for w in synth.split_rows_by_head(inp.Wo, nh, d, 4)]
    parts = []
    for r in range(2):
        ws = torch.empty(L.attn_partial_workspace_bytes(S, H, nh // 2, d, 2), dtype=torch.uint8, device="cuda")
        P = torch.empty(S, H, dtype=torch.float32, device="cuda")
        L.attn_partial_forward(X, Wq[2 * r:2 * r + 2], Wo[2 * r:2 * r + 2], nh // 2, d, P, ws)
        parts.append(P)
    Y, _ = _reduce_both_ways(parts, X, None, None, torch.float32)
    assert rel_err(Y, O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d)) <= TOL_BF16


def test_tp_sublayer_single_rank_on_gpu(cuda_device):
    """tp_dist.TPSublayer with one rank (no collective) runs the library's
    kernels end to end in both modes."""
    S, H, F = 256, 512, 2048
    inp = synth.gen_mlp(S, H, F, seed=3)
    X = inp.X.cuda()
    A = [a.cuda() for a in synth.split_columns(inp.A, 2)]
    B = [b.cuda() for b in synth.split_rows(inp.B, 2)]
    ws = torch.empty(L.mlp_partial_workspace_bytes(S, H, F, 2), dtype=torch.uint8, device="cuda")
    ref = O.mlp_block(inp.X, inp.A, inp.B)
    for mode in tp_dist.MODES:
        sub = tp_dist.TPSublayer(tp_dist.mlp_partial_fn(A, B, ws), S, H, torch.bfloat16, torch.bfloat16, mode=mode,
                                 device="cuda", world=1, rank=0)
        Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
        st = torch.cuda.Stream()
        sub.forward(X, Y, st)
        torch.cuda.synchronize()
        assert rel_err(Y, ref) <= TOL_BF16
