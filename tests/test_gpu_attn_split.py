"""The attention kernel's last-wave key split on the GPU.

Mode 2 splits every (head, 256 query rows) unit into two CTAs over the two
halves of the keys, so every warp's rows go through the claim / store / merge
path; mode 1 (the default) splits only the last partial wave.  Each is checked
against the fp64 oracle, against the unsplit kernel (mode 0), and run twice:
the merge is symmetric in the two halves, so the output must be bitwise the
same whichever half finished first.  The training forward's log2 row
denominators (what the backward rebuilds P from) go through the same merge and
are checked through the backward's gradients.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import synth
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu

TOL = 2e-2


def rel_err(got, ref) -> float:
    got = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / np.abs(ref).max())


@pytest.fixture
def split_mode():
    yield L.set_attn_kv_split
    L.set_attn_kv_split(1)


def _run(inp, nh, t, mode):
    d = 128
    L.set_attn_kv_split(mode)
    X = inp.X.cuda()
    S, H = X.shape
    Wq = [w.cuda() for w in synth.split_qkv_by_head(inp.Wqkv, nh, d, t)]
    Wo = [w.cuda() for w in synth.split_rows_by_head(inp.Wo, nh, d, t)]
    Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    # garbage in the workspace: stale flags must never be taken for this launch's
    ws = torch.full((L.attn_workspace_bytes(S, H, nh, d, t),), 0x5A, dtype=torch.uint8, device="cuda")
    L.attn_forward(X, Wq, Wo, nh, d, Y, ws)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    return Y


# (S, nh, t): an odd 128-row tile count (S = 384: the second tile of the last
# unit is not stored), key halves of one block each (S = 256), uneven halves
# (S = 640: 5 key blocks, 2 + 3), several shards.
@pytest.mark.parametrize("S,nh,t", [(256, 2, 1), (384, 2, 2), (640, 4, 4), (1024, 8, 2)])
def test_every_unit_split(cuda_device, split_mode, S, nh, t):
    d = 128
    inp = synth.gen_attn(S, nh * d, seed=S + 3 * nh)
    whole, split, _ = L.attn_split_plan(S, nh, mode=2)
    assert whole == 0 and split == nh * ((S + 255) // 256)
    Y2 = _run(inp, nh, t, 2)
    Y2b = _run(inp, nh, t, 2)
    Y0 = _run(inp, nh, t, 0)
    assert rel_err(Y2, O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d)) <= TOL
    assert torch.equal(Y2, Y2b)
    assert rel_err(Y2.float(), Y0.float().cpu().numpy()) <= 1e-2


def test_last_wave_split_default(cuda_device, split_mode):
    """S = 1024, 16 heads: 64 units on 148 SMs, all in one partial wave, so
    the default plan splits each into two (128 CTAs)."""
    S, nh, t, d = 1024, 16, 4, 128
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    whole, split, kv_half = L.attn_split_plan(S, nh, slots=sms, mode=1)
    assert (whole, split, kv_half) == (0, 64, 4)
    inp = synth.gen_attn(S, nh * d, seed=5)
    Y1 = _run(inp, nh, t, 1)
    rows = synth.row_sample(S, 6)
    assert rel_err(Y1[rows], O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d, rows=rows)) <= TOL
    assert torch.equal(Y1, _run(inp, nh, t, 1))


def test_split_rescale_inside_one_half(cuda_device, split_mode):
    """The last key block is 4x larger for rows 0..383 (the kernel rescales
    O in the second half only): the merge must weigh the two halves by their
    own running maxima."""
    d, nh, S = 128, 2, 512
    inp = synth.gen_attn(S, nh * d, seed=21)
    X = inp.X.float()
    X[384:] *= 4.0
    inp.X = X.to(torch.bfloat16)
    Y = _run(inp, nh, 2, 2)
    rows = list(range(384))
    ref = O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d, rows=rows)
    assert rel_err(Y[:384], ref) <= TOL


@pytest.mark.parametrize("S,nh,t", [(512, 4, 2), (384, 2, 1)])
def test_training_forward_split_gradients(cuda_device, split_mode, S, nh, t):
    """The merged log2 denominators feed the backward's softmax rebuild."""
    from test_gpu_attn_backward import run_and_check
    L.set_attn_kv_split(2)
    run_and_check(S, nh, t, seed=40 + S)
