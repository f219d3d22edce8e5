"""tp_mlp_forward_noalloc, the MLP entry point that allocates nothing: its
scratch is a fixed device array inside the library, for callers that cannot
allocate device memory (plugin hosts that forbid allocation in their execute
hook, latency-critical loops that cannot pay for cudaMalloc's implicit
synchronisation, programs whose own allocator holds the device memory).

Checked through the C ABI:
  * against tp_mlp_forward on the same inputs, bit for bit: both run the same
    deterministic kernels (fixed reduction order, plain stores into the
    partial-sum slots), so any difference would be a scratch layout, offset or
    stale-read error;
  * against the fp64 oracle, with the tolerance of the other bf16 parity tests;
  * on calls in a row that share the array: a larger call (more scratch, four
    K-split slots) first, then a smaller one whose slots sit at other offsets
    and must not pick up the larger call's leftovers, then the larger again.
This file is collected last so that a run stopping at its first failure has
already run every other test; it also passes on its own in a fresh process
(the first call on the device looks the array up)."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import synth
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
INVALID, WS_SMALL = 1, 3


def _rel(a, ref):
    a = np.asarray(a, dtype=np.float64)
    return float(np.abs(a - ref).max() / np.abs(ref).max())


class _Case:
    def __init__(self, S, H, F, t, seed):
        self.S, self.H, self.F, self.t = S, H, F, t
        inp = synth.gen_mlp(S, H, F, seed=seed)
        self.inp = inp
        self.X = inp.X.cuda()
        self.As = [a.cuda() for a in synth.split_columns(inp.A, t)]
        self.Bs = [b.cuda() for b in synth.split_rows(inp.B, t)]
        g = torch.Generator().manual_seed(seed + 1)
        self.gamma_h = 1.0 + 0.25 * torch.randn(H, generator=g)
        self.beta_h = 0.25 * torch.randn(H, generator=g)
        self.gamma, self.beta = self.gamma_h.cuda(), self.beta_h.cuda()

    def with_workspace(self):
        Y = torch.empty(self.S, self.H, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(L.mlp_workspace_bytes(self.S, self.H, self.F, self.t, torch.bfloat16), dtype=torch.uint8,
                         device="cuda")
        L.mlp_forward(self.X, self.As, self.Bs, Y, ws, gamma=self.gamma, beta=self.beta)
        torch.cuda.synchronize()
        return Y

    def noalloc(self):
        Y = torch.full((self.S, self.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        L.mlp_forward_noalloc(self.X, self.As, self.Bs, Y, gamma=self.gamma, beta=self.beta)
        torch.cuda.synchronize()
        assert L.device_error() == 0
        return Y

    def oracle(self, rows):
        return O.mlp_block(self.inp.X, self.inp.A, self.inp.B, gamma=self.gamma_h, beta=self.beta_h, rows=rows)


def test_noalloc_matches_workspace_entry_point_on_calls_in_a_row(cuda_device):
    cap = L.lib().tp_noalloc_scratch_bytes()
    big = _Case(1024, 1024, 4096, 4, seed=31)
    small = _Case(200, 512, 2048, 4, seed=37)
    for c in (big, small):
        assert L.mlp_workspace_bytes(c.S, c.H, c.F, c.t, torch.bfloat16) <= cap
    # the larger call cuts its row-split K loop into 4 f32 slots
    assert L.gemm_plan(big.S, big.t, 1, big.F // big.t, big.H, 1, max_splits=4)[1] == 4

    refs = {id(c): c.with_workspace() for c in (big, small)}
    rows_big = synth.row_sample(big.S, seed=32, n=64)
    oracle = {id(big): (rows_big, big.oracle(rows_big)), id(small): (list(range(small.S)), small.oracle(None))}
    for c in (big, small, big, small):
        Y = c.noalloc()
        assert torch.equal(Y, refs[id(c)]), "no-alloc result differs from tp_mlp_forward's"
        rows, ref = oracle[id(c)]
        assert _rel(Y[rows].double().cpu().numpy(), ref) <= TOL_BF16


def test_noalloc_first_call_may_be_empty(cuda_device):
    # S == 0 passes the argument checks, looks the array up and launches nothing
    c = _Case(128, 256, 1024, 2, seed=41)
    pa, ka = L._ptrs(c.As)
    pb, kb = L._ptrs(c.Bs)
    code = L.lib().tp_mlp_forward_noalloc(0, c.H, c.F, c.t, 1, 1, None, pa, pb, None, None, 1e-5, 1, None, None)
    assert code == 0
    Y = c.noalloc()
    assert torch.equal(Y, c.with_workspace())


def test_noalloc_rejects_sizes_beyond_its_scratch_after_the_argument_checks(cuda_device):
    cap = L.lib().tp_noalloc_scratch_bytes()
    S, H, F, t = 2048, 4096, 16384, 4
    assert L.mlp_workspace_bytes(S, H, F, t, torch.bfloat16) > cap
    X = torch.zeros(S, H, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(S, H, dtype=torch.bfloat16, device="cuda")
    A = [torch.zeros(H, F // t, dtype=torch.bfloat16, device="cuda") for _ in range(t)]
    B = [torch.zeros(F // t, H, dtype=torch.bfloat16, device="cuda") for _ in range(t)]
    pa, ka = L._ptrs(A)
    pb, kb = L._ptrs(B)
    Yc = ctypes.c_void_p(Y.data_ptr())
    Xc = ctypes.c_void_p(X.data_ptr())
    code = L.lib().tp_mlp_forward_noalloc(S, H, F, t, 1, 1, Xc, pa, pb, None, None, 1e-5, 1, Yc, None)
    assert code == WS_SMALL  # nothing launched
    torch.cuda.synchronize()
    assert not Y.any()
    # an oversized call with a bad argument reports the argument, as tp_mlp_forward would
    assert L.lib().tp_mlp_forward_noalloc(S, H, F, t, 1, 1, None, pa, pb, None, None, 1e-5, 1, Yc, None) == INVALID
    assert L.lib().tp_mlp_forward_noalloc(S, H, F, t, 1, 1, Xc, pa, pb, None, None, 1e-5, 9, Yc, None) == INVALID
