"""tp_mlp_forward_noalloc, the MLP entry point that allocates nothing: its
scratch is a fixed device array inside the library, for callers that cannot
allocate device memory (plugin hosts that forbid allocation in their execute
hook, latency-critical loops, programs whose own allocator holds the device
memory).  Checked through the C ABI against tp_mlp_forward, on two calls in a
row, with the tolerance of the other bf16 parity tests.  This file is
collected last so that a run stopping at its first failure has already run
every other test."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import synth

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.abs(a - b).max() / np.abs(b).max())


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    S, H, F, t = 200, 512, 2048, 4
    inp = synth.gen_mlp(S, H, F, seed=31)
    X = inp.X.cuda()
    As = [a.cuda() for a in synth.split_columns(inp.A, t)]
    Bs = [b.cuda() for b in synth.split_rows(inp.B, t)]
    gamma = torch.randn(H, generator=torch.Generator().manual_seed(1)).cuda()
    beta = torch.randn(H, generator=torch.Generator().manual_seed(2)).cuda()
    assert L.mlp_workspace_bytes(S, H, F, t, torch.bfloat16) <= L.lib().tp_noalloc_scratch_bytes()

    ref = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.mlp_workspace_bytes(S, H, F, t, torch.bfloat16), dtype=torch.uint8, device="cuda")
    L.mlp_forward(X, As, Bs, ref, ws, gamma=gamma, beta=beta)
    torch.cuda.synchronize()

    for _ in range(2):
        Y = torch.full((S, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        L.mlp_forward_noalloc(X, As, Bs, Y, gamma=gamma, beta=beta)
        torch.cuda.synchronize()
        assert L.device_error() == 0
        assert torch.isfinite(Y.float()).all()
        assert _rel(Y, ref) <= TOL_BF16


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    cap = L.lib().tp_noalloc_scratch_bytes()
    S, H, F, t = 2048, 4096, 16384, 4
    assert L.mlp_workspace_bytes(S, H, F, t, torch.bfloat16) > cap
    pa = (ctypes.c_void_p * t)(*([0x10000] * t))
    pp = ctypes.cast(pa, ctypes.POINTER(ctypes.c_void_p))
    code = L.lib().tp_mlp_forward_noalloc(S, H, F, t, 1, 1, ctypes.c_void_p(0x10000), pp, pp, None, None, 1e-5, 1,
                                          ctypes.c_void_p(0x10000), None)
    assert code == 3  # TP_ERR_WORKSPACE_TOO_SMALL, nothing launched
