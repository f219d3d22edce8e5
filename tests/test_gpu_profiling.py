"""The library's launch counting and event sampling (what bench.py's
per-kernel numbers rest on): every launch made while profiling is enabled is
counted, events are recorded only while sampling is on, and the timed
durations are positive."""
from __future__ import annotations

import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import synth

pytestmark = pytest.mark.gpu


def test_profile_counts_every_launch_and_times_sampled_ones(cuda_device):
    inp = synth.gen_mlp(256, 512, 2048, seed=0)
    X = inp.X.cuda()
    As = [a.cuda() for a in synth.split_columns(inp.A, 4)]
    Bs = [b.cuda() for b in synth.split_rows(inp.B, 4)]
    Y = torch.empty_like(X)
    ws = torch.empty(L.mlp_workspace_bytes(256, 512, 2048, 4, torch.bfloat16), dtype=torch.uint8, device="cuda")
    L.profile_enable(True)
    try:
        for i in range(6):
            L.profile_sample(i % 3 == 0)  # steps 0 and 3
            L.mlp_forward(X, As, Bs, Y, ws)
        torch.cuda.synchronize()
        prof = L.profile_collect()
    finally:
        L.profile_enable(False)
    gemm = prof["gemm_tcgen05"]
    ln = prof["reduce_residual_layernorm"]
    assert gemm[0] == 12 and ln[0] == 6          # launches: 2 GEMMs + 1 LayerNorm per step
    assert gemm[1] == 4 and ln[1] == 2           # timed: the two sampled steps only
    assert gemm[2] > 0.0 and ln[2] > 0.0
    # collect cleared the record
    L.profile_enable(True)
    L.profile_enable(False)
    assert all(v[0] == 0 for v in L.profile_collect().values())
