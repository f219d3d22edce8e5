"""Failure detection on the GPU without a fault: a bounded device-side wait
that nothing completes gives up, raises the library's device error word, and
returns control; the host reads TP_ERR_TIMEOUT and the context keeps working."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import synth
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu

TP_ERR_TIMEOUT = 5


def test_bounded_wait_times_out_and_context_survives(cuda_device):
    assert L.device_error() == 0
    L.selftest_wait_timeout(20_000_000)  # ~10 ms of SM cycles
    torch.cuda.synchronize()
    assert L.device_error() == TP_ERR_TIMEOUT
    assert L.device_error() == 0  # reading clears it
    # the library still computes correctly afterwards
    inp = synth.gen_mlp(128, 256, 512, seed=2)
    X = inp.X.cuda()
    Y = torch.empty_like(X)
    ws = torch.empty(L.mlp_workspace_bytes(128, 256, 512, 2, torch.bfloat16), dtype=torch.uint8, device="cuda")
    L.mlp_forward(X, [a.cuda() for a in synth.split_columns(inp.A, 2)],
                  [b.cuda() for b in synth.split_rows(inp.B, 2)], Y, ws)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    ref = O.mlp_block(inp.X, inp.A, inp.B)
    assert np.abs(Y.double().cpu().numpy() - ref).max() / np.abs(ref).max() <= 2e-2


def test_selftest_rejects_bad_limit(cuda_device):
    with pytest.raises(L.TPError):
        L.selftest_wait_timeout(0)


def test_bounded_flag_wait_times_out_and_context_survives(cuda_device):
    """The stream-K finisher's kind of wait (a global flag another CTA pair
    publishes): a flag nothing sets makes it give up with TP_ERR_TIMEOUT."""
    assert L.device_error() == 0
    L.selftest_flag_wait_timeout(20_000_000)
    torch.cuda.synchronize()
    assert L.device_error() == TP_ERR_TIMEOUT
    assert L.device_error() == 0
    with pytest.raises(L.TPError):
        L.selftest_flag_wait_timeout(0)
