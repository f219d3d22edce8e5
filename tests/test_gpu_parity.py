"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Error metric: max|GPU - oracle| / max|oracle| over the compared elements.
Bar: <= 2e-2 for bf16 storage with f32 accumulation, <= 1e-4 for f32.
Small cases are compared element by element in full (several tiles plus a
ragged tail in every dimension the kernels tile); the full-size workloads are
run in the same launch configuration the benchmark times and compared on a
deterministic sample of rows (every output row depends only on its own input
row for the MLP, and on all K/V rows for attention, which the oracle computes
in full).
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

TOL_BF16 = 2e-2
TOL_F32 = 1e-4


def rel_err(got, ref) -> float:
    got = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / np.abs(ref).max())


def _dev(ts):
    return [t.cuda() for t in ts]


def run_mlp(inp, t, out_dtype=None, act="gelu_tanh", gamma=None, beta=None):
    X = inp.X.cuda()
    S, H = X.shape
    F = inp.A.shape[1]
    As = _dev(synth.split_columns(inp.A, t))
    Bs = _dev(synth.split_rows(inp.B, t))
    out_dtype = out_dtype or X.dtype
    Y = torch.empty(S, H, dtype=out_dtype, device="cuda")
    ws = torch.empty(max(1, L.mlp_workspace_bytes(S, H, F, t, X.dtype)), dtype=torch.uint8, device="cuda")
    g = None if gamma is None else gamma.cuda()
    b = None if beta is None else beta.cuda()
    L.mlp_forward(X, As, Bs, Y, ws, gamma=g, beta=b, act=act)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    return Y


def run_attn(inp, nh, d, t, out_dtype=torch.bfloat16):
    X = inp.X.cuda()
    S, H = X.shape
    Wq = _dev(synth.split_qkv_by_head(inp.Wqkv, nh, d, t))
    Wo = _dev(synth.split_rows_by_head(inp.Wo, nh, d, t))
    Y = torch.empty(S, H, dtype=out_dtype, device="cuda")
    ws = torch.empty(L.attn_workspace_bytes(S, H, nh, d, t), dtype=torch.uint8, device="cuda")
    L.attn_forward(X, Wq, Wo, nh, d, Y, ws)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    return Y


# ------------------------------------------------------------- MLP, small

@pytest.mark.parametrize("t", [1, 2, 4])
def test_mlp_tiny_f32_full(cuda_device, t):
    w = WORKLOADS["mlp_tiny_f32"]
    inp = synth.gen_mlp(w.S, w.H, w.F, seed=w.seed, dtype=torch.float32)
    Y = run_mlp(inp, t)
    ref = O.mlp_block(inp.X, inp.A, inp.B, eps=1e-5)
    assert rel_err(Y, ref) <= TOL_F32


@pytest.mark.parametrize("act", ["gelu_tanh", "gelu_erf", "relu", "none"])
def test_mlp_f32_ragged_acts(cuda_device, act):
    inp = synth.gen_mlp(77, 136, 3 * 104, seed=3, dtype=torch.float32)
    Y = run_mlp(inp, 3, act=act)
    assert rel_err(Y, O.mlp_block(inp.X, inp.A, inp.B, act=act)) <= TOL_F32


@pytest.mark.parametrize("S,H,F,t", [
    (256, 256, 1024, 2),     # whole tiles
    (200, 264, 1200, 3),     # ragged rows, ragged K (264 = 4*64 + 8), shard width 400 (ragged N tile)
    (129, 512, 2048, 8),     # one row past a tile, 8 shards of 256
    (1, 64, 64, 1),          # single row, single partial tile
])
def test_mlp_bf16_small_full(cuda_device, S, H, F, t):
    inp = synth.gen_mlp(S, H, F, seed=S + H, dtype=torch.bfloat16)
    Y = run_mlp(inp, t)
    assert rel_err(Y, O.mlp_block(inp.X, inp.A, inp.B)) <= TOL_BF16


@pytest.mark.parametrize("act", ["gelu_erf", "relu", "none"])
def test_mlp_bf16_acts_f32_out_gamma_beta(cuda_device, act):
    inp = synth.gen_mlp(192, 384, 1536, seed=5, dtype=torch.bfloat16)
    g = torch.randn(384, generator=torch.Generator().manual_seed(1))
    b = torch.randn(384, generator=torch.Generator().manual_seed(2))
    Y = run_mlp(inp, 2, out_dtype=torch.float32, act=act, gamma=g, beta=b)
    assert rel_err(Y, O.mlp_block(inp.X, inp.A, inp.B, g, b, act=act)) <= TOL_BF16


def test_mlp_deterministic_and_t_invariant(cuda_device):
    inp = synth.gen_mlp(256, 512, 2048, seed=11, dtype=torch.bfloat16)
    ys = {t: run_mlp(inp, t) for t in (1, 2, 4, 8)}
    again = run_mlp(inp, 4)
    assert torch.equal(ys[4], again), "repeated runs must be bitwise equal"
    ref = O.mlp_block(inp.X, inp.A, inp.B)
    for t, y in ys.items():
        assert rel_err(y, ref) <= TOL_BF16, t
        assert rel_err(y, ys[1].double().cpu().numpy()) <= TOL_BF16, t


def test_mlp_empty_rows(cuda_device):
    inp = synth.gen_mlp(1, 64, 128, seed=0)
    X = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    Y = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    L.mlp_forward(X, _dev(synth.split_columns(inp.A, 2)), _dev(synth.split_rows(inp.B, 2)), Y, ws)
    Xl = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    Yl = torch.empty(0, 128, dtype=torch.float32, device="cuda")
    L.linear_column_forward(Xl, _dev(synth.split_columns(inp.A, 2)), Yl)
    torch.cuda.synchronize()


def test_mlp_split_direction_swapped_fails_parity(cuda_device):
    """Row-splitting A and column-splitting B (the swapped wiring) is not the
    sublayer: it must either be rejected or miss the oracle."""
    inp = synth.gen_mlp(128, 256, 512, seed=4, dtype=torch.bfloat16)
    # Give the kernel A's row shards as if they were column shards: same byte
    # counts, wrong partition.
    wrongA = [a.reshape(256, 256).contiguous() for a in synth.split_rows(inp.A, 2)]
    X = inp.X.cuda()
    Y = torch.empty(128, 256, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.mlp_workspace_bytes(128, 256, 512, 2, torch.bfloat16), dtype=torch.uint8, device="cuda")
    L.mlp_forward(X, _dev(wrongA), _dev(synth.split_rows(inp.B, 2)), Y, ws)
    torch.cuda.synchronize()
    assert rel_err(Y, O.mlp_block(inp.X, inp.A, inp.B)) > TOL_BF16


# ------------------------------------------------------------ linears

@pytest.mark.parametrize("t", [1, 2, 4])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_linear_column_small(cuda_device, t, out):
    inp = synth.gen_linear(300, 328, 8 * 3 * 40, seed=t)
    X = inp.X.cuda()
    Y = torch.empty(300, inp.W.shape[1], dtype=out, device="cuda")
    L.linear_column_forward(X, _dev(synth.split_columns(inp.W, t)), Y)
    torch.cuda.synchronize()
    assert rel_err(Y, O.linear_column(inp.X, inp.W)) <= TOL_BF16


@pytest.mark.parametrize("t", [1, 2, 4])
def test_linear_row_small(cuda_device, t):
    inp = synth.gen_linear(300, 4 * 136, 520, seed=t)
    X = inp.X.cuda()
    Y = torch.empty(300, 520, dtype=torch.float32, device="cuda")
    L.linear_row_forward(X, _dev(synth.split_rows(inp.W, t)), Y)
    torch.cuda.synchronize()
    assert rel_err(Y, O.linear_row(inp.X, inp.W)) <= TOL_BF16


def test_linears_f32(cuda_device):
    inp = synth.gen_linear(70, 96, 160, seed=1, dtype=torch.float32)
    X = inp.X.cuda()
    Y = torch.empty(70, 160, dtype=torch.float32, device="cuda")
    L.linear_column_forward(X, _dev(synth.split_columns(inp.W, 2)), Y, act="gelu_tanh")
    torch.cuda.synchronize()
    assert rel_err(Y, O.linear_column(inp.X, inp.W, act="gelu_tanh")) <= TOL_F32
    L.linear_row_forward(X, _dev(synth.split_rows(inp.W, 4)), Y)
    torch.cuda.synchronize()
    assert rel_err(Y, O.linear_row(inp.X, inp.W)) <= TOL_F32


@pytest.mark.parametrize("kind", ["linear_col_4096x4096x8192", "linear_row_4096x4096x8192"])
@pytest.mark.parametrize("t", [1, 2, 4])
def test_linear_full_size(cuda_device, kind, t):
    w = WORKLOADS[kind]
    inp = synth.gen_linear(w.M, w.K, w.N, seed=w.seed)
    X = inp.X.cuda()
    Y = torch.empty(w.M, w.N, dtype=torch.float32, device="cuda")
    if w.kind == "linear_col":
        L.linear_column_forward(X, _dev(synth.split_columns(inp.W, t)), Y)
    else:
        L.linear_row_forward(X, _dev(synth.split_rows(inp.W, t)), Y)
    torch.cuda.synchronize()
    rows = synth.row_sample(w.M, w.seed + 1)
    assert rel_err(Y[rows], O.linear_column(inp.X, inp.W, rows=rows)) <= TOL_BF16


# ------------------------------------------------------ reduce + LayerNorm

# H: one warp per row (8, 264), the one-CTA rows with the next row group's
# loads issued ahead at two and four chunks per thread, ragged (2056, 4104)
# and whole (4096, 8192), and the 12- and 16-warp rows.
@pytest.mark.parametrize("H", [8, 264, 2056, 4096, 4104, 8192, 12288, 16384])
@pytest.mark.parametrize("nparts", [0, 1, 3])
def test_reduce_residual_layernorm(cuda_device, H, nparts):
    g = torch.Generator().manual_seed(H + nparts)
    S = 37
    X = torch.randn(S, H, generator=g).to(torch.bfloat16)
    P = torch.randn(max(nparts, 1), S, H, generator=g) * 3.0
    gam = torch.randn(H, generator=g)
    bet = torch.randn(H, generator=g)
    Y = torch.empty(S, H, dtype=torch.float32, device="cuda")
    L.reduce_residual_layernorm(P[:nparts].cuda() if nparts else None, X.cuda(), Y, gam.cuda(), bet.cuda())
    torch.cuda.synchronize()
    Z = X.double().numpy() + (P[:nparts].double().numpy().sum(0) if nparts else 0.0)
    assert rel_err(Y, O.layernorm(Z, gam, bet)) <= TOL_F32


@pytest.mark.parametrize("H", [2056, 4104])
def test_reduce_residual_layernorm_bf16_out(cuda_device, H):
    """The sublayers' case: one f32 partial, bf16 X and bf16 Y, rows whose
    chunk count does not fill the CTA (the look-ahead kernel's bounds)."""
    g = torch.Generator().manual_seed(H)
    S = 53
    X = torch.randn(S, H, generator=g).to(torch.bfloat16)
    P = torch.randn(1, S, H, generator=g) * 3.0
    gam = torch.randn(H, generator=g)
    bet = torch.randn(H, generator=g)
    Y = torch.empty(S, H, dtype=torch.bfloat16, device="cuda")
    L.reduce_residual_layernorm(P.cuda(), X.cuda(), Y, gam.cuda(), bet.cuda())
    torch.cuda.synchronize()
    Z = X.double().numpy() + P.double().numpy().sum(0)
    assert rel_err(Y, O.layernorm(Z, gam, bet)) <= TOL_BF16


# --------------------------------------------------------------- attention

@pytest.mark.parametrize("S,nh,t", [(128, 1, 1), (256, 4, 2), (384, 4, 4), (512, 8, 8)])
def test_attention_small_full(cuda_device, S, nh, t):
    d = 128
    inp = synth.gen_attn(S, nh * d, seed=S + nh)
    Y = run_attn(inp, nh, d, t)
    assert rel_err(Y, O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d)) <= TOL_BF16


def test_attention_late_large_keys_rescale(cuda_device):
    """Keys of the last 128-key block are 4x larger, so for the unscaled query
    rows 0..383 that block's row max exceeds the running max by more than the
    lazy-rescale threshold (2^8): the O accumulator is rescaled in TMEM."""
    d, nh, S = 128, 2, 512
    inp = synth.gen_attn(S, nh * d, seed=21)
    X = inp.X.float()
    X[384:] *= 4.0
    inp.X = X.to(torch.bfloat16)
    Y = run_attn(inp, nh, d, 2)
    rows = list(range(384))
    ref = O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d, rows=rows)
    assert rel_err(Y[:384], ref) <= TOL_BF16


# ------------------------------------------------------ full-size workloads

@pytest.mark.slow
@pytest.mark.parametrize("t", [4, 1, 2, 8])
def test_mlp_s2048_h4096_f16384(cuda_device, t):
    w = WORKLOADS["mlp_s2048_h4096_f16384"]
    inp = _cached_mlp(w)
    Y = run_mlp(inp, t)
    rows = synth.row_sample(w.S, w.seed + 1)
    assert rel_err(Y[rows], O.mlp_block(inp.X, inp.A, inp.B, rows=rows)) <= TOL_BF16


@pytest.mark.slow
@pytest.mark.parametrize("t", [4, 1, 2, 8])
def test_attn_s2048_h8192(cuda_device, t):
    w = WORKLOADS["attn_s2048_h8192_64x128"]
    if w.name not in _CACHE:  # inputs and the oracle's 64 sampled rows, shared by every t
        inp = synth.gen_attn(w.S, w.H, seed=w.seed)
        rows = synth.row_sample(w.S, w.seed + 1)
        _CACHE[w.name] = (inp, rows, O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, w.nh, w.d, rows=rows))
    inp, rows, ref = _CACHE[w.name]
    Y = run_attn(inp, w.nh, w.d, t)
    assert len(rows) == 64
    assert rel_err(Y[rows], ref) <= TOL_BF16


@pytest.mark.slow
def test_mlp_s4096_h12288_f49152(cuda_device):
    w = WORKLOADS["mlp_s4096_h12288_f49152"]
    inp = synth.gen_mlp(w.S, w.H, w.F, seed=w.seed)
    Y = run_mlp(inp, w.t)
    rows = synth.row_sample(w.S, w.seed + 1)
    assert len(rows) == 64  # rows 0 and S-1 and 62 drawn; they fall in all 16 of the 256-row tiles
    assert rel_err(Y[rows], O.mlp_block(inp.X, inp.A, inp.B, rows=rows)) <= TOL_BF16


_CACHE = {}


def _cached_mlp(w):
    if w.name not in _CACHE:
        _CACHE[w.name] = synth.gen_mlp(w.S, w.H, w.F, seed=w.seed)
    return _CACHE[w.name]


# --------------------------------------------------------- Transformer block

@pytest.mark.parametrize("pre_ln", [False, True])
@pytest.mark.parametrize("S,nh,F,t", [(256, 2, 1024, 2), (384, 4, 2048, 4)])
@pytest.mark.parametrize("layout", ["in_out", "out_in"])
def test_transformer_block(cuda_device, pre_ln, S, nh, F, t, layout):
    d = 128
    tr = (lambda ws: [w.t().contiguous() for w in ws]) if layout == "out_in" else (lambda ws: ws)
    H = nh * d
    a = synth.gen_attn(S, H, seed=S + 1)
    m = synth.gen_mlp(S, H, F, seed=S + 2)
    g = torch.Generator().manual_seed(3)
    ln1 = (torch.randn(H, generator=g) * 0.2 + 1.0, torch.randn(H, generator=g) * 0.1)
    ln2 = (torch.randn(H, generator=g) * 0.2 + 1.0, torch.randn(H, generator=g) * 0.1)
    X = a.X.cuda()
    Y = torch.empty(S, H, dtype=torch.float32, device="cuda")
    ws = torch.empty(L.block_workspace_bytes(S, H, F, nh, d, t), dtype=torch.uint8, device="cuda")
    L.block_forward(X, _dev(tr(synth.split_qkv_by_head(a.Wqkv, nh, d, t))),
                    _dev(tr(synth.split_rows_by_head(a.Wo, nh, d, t))), _dev(tr(synth.split_columns(m.A, t))),
                    _dev(tr(synth.split_rows(m.B, t))), nh, d, Y, ws, pre_ln=pre_ln,
                    ln1=(ln1[0].cuda(), ln1[1].cuda()), ln2=(ln2[0].cuda(), ln2[1].cuda()), layout=layout)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    ref = O.transformer_block(a.X, a.Wqkv, a.Wo, m.A, m.B, nh, d, ln1=ln1, ln2=ln2, pre_ln=pre_ln)
    assert rel_err(Y, ref) <= TOL_BF16


@pytest.mark.parametrize("form,bound,at0", [(0, 3.0e-6, 0.99999928), (1, 7.6e-5, 0.999928057)])
def test_attention_polynomial_exp2_against_exp2f(cuda_device, form, bound, at0):
    """Part of the attention softmax's exponentials can be evaluated on the
    FMA pipe.  Over the range its arguments take (s * log2(e)/sqrt(d) - m, at
    most 2^8 above the running max, far below it for small scores), the
    relative error against CUDA's exp2f stays within the polynomial's fitted
    minimax bound (2.7e-6 for degree 4, 7.5e-5 for the degree-3 pair form)
    plus exp2f's own few ulp; both lanes of the pair form are checked (the
    inputs alternate between them)."""
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_001), torch.linspace(-1.0, 1.0, 200_001),
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 8.0, -125.0, 3.25])]).cuda()
    yp, yr = L.selftest_exp2(x, form=form)
    torch.cuda.synchronize()
    rel = ((yp.double() - yr.double()).abs() / yr.double()).max().item()
    assert rel <= bound, rel
    # integer arguments: 2^n times the polynomial's value at f = 0, exactly
    yi, _ = L.selftest_exp2(torch.tensor([0.0, 1.0, -3.0, 7.0]).cuda(), form=form)
    torch.cuda.synchronize()
    want = np.float32(at0) * np.array([1.0, 2.0, 0.125, 128.0], dtype=np.float32)
    np.testing.assert_array_equal(yi.cpu().numpy(), want)
