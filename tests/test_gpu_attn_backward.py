"""GPU parity of the attention sublayer's backward pass (tp_attn_forward_train
+ tp_attn_backward) against the fp64 oracle's chain-rule gradients.

dX is compared whole; each shard's dWqkv_s and dWo_s against the oracle's
dWqkv / dWo cut the way the weights are (by head); dgamma and dbeta whole.
Same metric and bar as the forward (max|GPU - oracle| / max|oracle| <= 2e-2).
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


def run_and_check(S, nh, t, seed, d=128):
    H = nh * d
    inp = synth.gen_attn(S, H, seed=seed)
    dY, g, b = synth.gen_upstream(S, H, seed=seed + 1)
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
    assert rel_err(Y, O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d, g, b)) <= TOL
    ref = O.attention_sublayer_backward(inp.X, inp.Wqkv, inp.Wo, nh, d, dY, g, b)
    ref_q = synth.split_qkv_by_head(torch.from_numpy(ref["dWqkv"]), nh, d, t)
    ref_o = synth.split_rows_by_head(torch.from_numpy(ref["dWo"]), nh, d, t)
    errs = {"dX": rel_err(dX, ref["dX"]), "dgamma": rel_err(dg, ref["dgamma"]), "dbeta": rel_err(db, ref["dbeta"])}
    for s in range(t):
        errs[f"dWqkv{s}"] = rel_err(dWq[s], ref_q[s].numpy())
        errs[f"dWo{s}"] = rel_err(dWo[s], ref_o[s].numpy())
    assert all(e <= TOL for e in errs.values()), errs


# The per-head GEMMs run over groups of up to 8 heads per launch: (256, 12, 4)
# and (512, 10, 2) end on a partial group, with the group's heads spread over
# several shards.  S = 128 runs the score tiles on single CTAs instead of pairs.
@pytest.mark.parametrize("S,nh,t", [(256, 2, 1), (384, 4, 2), (256, 4, 4), (512, 8, 2), (256, 12, 4),
                                    (512, 10, 2), (128, 2, 2)])
def test_attention_backward_small(cuda_device, S, nh, t):
    run_and_check(S, nh, t, seed=S + nh + t)


def test_attention_backward_group_of_seven(cuda_device):
    """S = 5888: eight heads' [S, S] P and dS matrices would pass 1 GiB, so the
    heads go through as a group of 7 and a group of 1."""
    run_and_check(5888, 8, 2, seed=11)


@pytest.mark.slow
def test_attention_backward_s2048_h8192(cuda_device):
    w = WORKLOADS["attn_s2048_h8192_64x128"]
    run_and_check(w.S, w.nh, w.t, seed=w.seed)
