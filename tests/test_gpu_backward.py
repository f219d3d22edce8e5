"""GPU parity of the MLP sublayer's backward pass (tp_mlp_forward_train +
tp_mlp_backward) against the fp64 oracle's chain-rule gradients.

Every gradient is compared as a whole tensor: dX [S, H]; dA and dB as the
concatenation of the per-shard gradients (column blocks of dA, row blocks of
dB: each shard's weight gradient stays with its shard); dgamma and dbeta.
Same metric and bar as the forward (max|GPU - oracle| / max|oracle| <= 2e-2):
the GPU keeps U, G, dZ and dU in bf16 and accumulates in f32.
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

TOL = 2e-2


def rel_err(got, ref) -> float:
    got = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / np.abs(ref).max())


def run_train_step(inp, t, dY, gamma, beta, act="gelu_tanh", layout="in_out"):
    X = inp.X.cuda()
    S, H = X.shape
    F = inp.A.shape[1]
    oi = layout == "out_in"
    As = [(a.t().contiguous() if oi else a).cuda() for a in synth.split_columns(inp.A, t)]
    Bs = [(b.t().contiguous() if oi else b).cuda() for b in synth.split_rows(inp.B, t)]
    g, b = gamma.cuda(), beta.cuda()
    Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    state = torch.empty(L.mlp_train_state_bytes(S, H, F, t), dtype=torch.uint8, device="cuda")
    L.mlp_forward_train(X, As, Bs, Y, state, gamma=g, beta=b, act=act, layout=layout)
    dX = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    dAs = [torch.empty(*(a.shape), dtype=torch.float32, device="cuda") for a in As]
    dBs = [torch.empty(*(b.shape), dtype=torch.float32, device="cuda") for b in Bs]
    dg = torch.empty(H, dtype=torch.float32, device="cuda")
    db = torch.empty(H, dtype=torch.float32, device="cuda")
    ws = torch.empty(L.mlp_backward_workspace_bytes(S, H, F, t), dtype=torch.uint8, device="cuda")
    L.mlp_backward(X, As, Bs, state, dY.cuda(), dX, dAs, dBs, ws, gamma=g, dgamma=dg, dbeta=db, act=act,
                   layout=layout)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    if oi:  # back to the [in, out] orientation the oracle uses
        dAs = [d.t() for d in dAs]
        dBs = [d.t() for d in dBs]
    return {"Y": Y, "dX": dX, "dA": torch.cat(dAs, dim=1), "dB": torch.cat(dBs, dim=0), "dgamma": dg, "dbeta": db}


def check(out, inp, dY, gamma, beta, act="gelu_tanh"):
    ref = O.mlp_block_backward(inp.X, inp.A, inp.B, dY, gamma, beta, act=act)
    errs = {k: rel_err(out[k], ref[k]) for k in ("dX", "dA", "dB", "dgamma", "dbeta")}
    assert all(e <= TOL for e in errs.values()), errs
    assert rel_err(out["Y"], O.mlp_block(inp.X, inp.A, inp.B, gamma, beta, act=act)) <= TOL
    return errs


@pytest.mark.parametrize("S,H,F,t", [
    (256, 256, 1024, 2),
    (300, 264, 1200, 3),     # ragged rows (also the K of the weight-gradient GEMMs), ragged K, shard width 400
    (129, 512, 2048, 8),
    (520, 1000, 2016, 2),
    (72, 6144, 1024, 2),     # LayerNorm backward with 2 chunks per thread
    (40, 12288, 512, 1),     # 3 chunks per thread (one row in flight)
    (24, 16384, 256, 1),     # 4 chunks per thread, the largest row
    (64, 64, 256, 2),        # every GEMM in single-CTA form (M <= 128), M-major A included
    (130, 64, 512, 2),       # weight gradients single-CTA, dU / dX in CTA pairs with a ragged tile
])
def test_backward_small(cuda_device, S, H, F, t):
    inp = synth.gen_mlp(S, H, F, seed=S + F, dtype=torch.bfloat16)
    dY, g, b = synth.gen_upstream(S, H, seed=S)
    check(run_train_step(inp, t, dY, g, b), inp, dY, g, b)


@pytest.mark.parametrize("S,H,F,t", [(256, 256, 1024, 2), (300, 264, 1200, 3), (64, 64, 256, 2)])
def test_backward_out_in_layout(cuda_device, S, H, F, t):
    """nn.Linear [out, in] weights and gradients: the M-split and per-shard
    weight-gradient paths with the operands' roles swapped."""
    inp = synth.gen_mlp(S, H, F, seed=S + 7, dtype=torch.bfloat16)
    dY, g, b = synth.gen_upstream(S, H, seed=S + 8)
    check(run_train_step(inp, t, dY, g, b, layout="out_in"), inp, dY, g, b)


@pytest.mark.parametrize("act", ["gelu_erf", "relu", "none"])
def test_backward_activations(cuda_device, act):
    inp = synth.gen_mlp(384, 512, 1536, seed=2, dtype=torch.bfloat16)
    dY, g, b = synth.gen_upstream(384, 512, seed=3)
    check(run_train_step(inp, 2, dY, g, b, act=act), inp, dY, g, b, act=act)


@pytest.mark.parametrize("tile_n", [480, 512])
def test_backward_wide_tiles(cuda_device, tile_n):
    inp = synth.gen_mlp(520, 1000, 2016, seed=5, dtype=torch.bfloat16)
    dY, g, b = synth.gen_upstream(520, 1000, seed=6)
    try:
        L.set_gemm_tile_n(tile_n)
        out = run_train_step(inp, 2, dY, g, b)
    finally:
        L.set_gemm_tile_n(0)
    check(out, inp, dY, g, b)


def test_backward_deterministic_and_forward_matches(cuda_device):
    inp = synth.gen_mlp(256, 512, 2048, seed=8, dtype=torch.bfloat16)
    dY, g, b = synth.gen_upstream(256, 512, seed=9)
    a1 = run_train_step(inp, 4, dY, g, b)
    a2 = run_train_step(inp, 4, dY, g, b)
    for k in a1:
        assert torch.equal(a1[k], a2[k]), k
    # the training forward's Y is the inference forward's Y
    X = inp.X.cuda()
    Y = torch.empty(256, 512, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.mlp_workspace_bytes(256, 512, 2048, 4, X.dtype), dtype=torch.uint8, device="cuda")
    L.mlp_forward(X, [a.cuda() for a in synth.split_columns(inp.A, 4)],
                  [x.cuda() for x in synth.split_rows(inp.B, 4)], Y, ws, gamma=g.cuda(), beta=b.cuda())
    torch.cuda.synchronize()
    assert rel_err(a1["Y"], Y.double().cpu().numpy()) <= 1e-2


def test_backward_t_invariant(cuda_device):
    inp = synth.gen_mlp(256, 512, 2048, seed=10, dtype=torch.bfloat16)
    dY, g, b = synth.gen_upstream(256, 512, seed=11)
    outs = {t: run_train_step(inp, t, dY, g, b) for t in (1, 2, 8)}
    for t in (2, 8):
        for k in ("dX", "dA", "dB", "dgamma", "dbeta"):
            assert rel_err(outs[t][k], outs[1][k].double().cpu().numpy()) <= TOL, (t, k)


@pytest.mark.slow
def test_backward_s2048_h4096_f16384(cuda_device):
    w = WORKLOADS["mlp_s2048_h4096_f16384"]
    inp = synth.gen_mlp(w.S, w.H, w.F, seed=w.seed)
    dY, g, b = synth.gen_upstream(w.S, w.H, seed=w.seed + 2)
    check(run_train_step(inp, w.t, dY, g, b), inp, dY, g, b)
