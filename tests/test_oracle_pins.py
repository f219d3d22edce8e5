"""Pins of the fp64 oracle to things other than itself.

Each check below ties one oracle function to a brute-force exact computation
(Python Fractions on small integer inputs), a closed form, an invariant, or an
independent library routine (scipy / torch fp64 CPU).  The planted-mistake
tests at the end swap a plausible error into the oracle (on the CPU) and assert
that at least one pin then fails, so the pins are known to have teeth.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import tp_oracle as O
from megatron_tensor_transformer_gelu_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# ------------------------------------------------------------------ helpers

def _exact_matmul(A, B):
    """Textbook triple loop over Fractions (exact)."""
    n, k = len(A), len(A[0])
    m = len(B[0])
    assert len(B) == k
    return [[sum((A[i][p] * B[p][j] for p in range(k)), Fraction(0)) for j in range(m)]
            for i in range(n)]


def _to_frac(M):
    return [[Fraction(int(v)) for v in row] for row in np.asarray(M)]


def _relu_frac(M):
    return [[v if v > 0 else Fraction(0) for v in row] for row in M]


def _small_int_case(seed, S, H, F, lo=-3, hi=4):
    rng = np.random.default_rng(seed)
    X = rng.integers(lo, hi, size=(S, H)).astype(np.float64)
    A = rng.integers(lo, hi, size=(H, F)).astype(np.float64)
    B = rng.integers(lo, hi, size=(F, H)).astype(np.float64)
    return X, A, B


# ------------------------------------------------------------------- checks
# Each check_* raises AssertionError when the oracle is wrong.

def check_gelu_library():
    u = np.linspace(-8.0, 8.0, 4001)
    ut = torch.from_numpy(u)
    ref_tanh = torch.nn.functional.gelu(ut, approximate="tanh").numpy()
    ref_erf = torch.nn.functional.gelu(ut).numpy()
    from scipy.stats import norm
    np.testing.assert_allclose(O.gelu_tanh(u), ref_tanh, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(O.gelu_erf(u), ref_erf, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(O.gelu_erf(u), u * norm.cdf(u), rtol=1e-12, atol=1e-15)


def check_gelu_identities():
    u = np.linspace(-6.0, 6.0, 1201)
    for g in (O.gelu_tanh, O.gelu_erf):
        # x*s(x) with s(x) + s(-x) = 1  =>  g(u) - g(-u) = u
        np.testing.assert_allclose(g(u) - g(-u), u, rtol=0, atol=1e-13)
        assert g(np.array([0.0]))[0] == 0.0
        np.testing.assert_allclose(g(np.array([30.0])), [30.0], rtol=1e-15)
        assert abs(g(np.array([-30.0]))[0]) < 1e-15
    # the tanh form approximates u*Phi(u) to within 4.74e-4 everywhere
    w = np.linspace(-12, 12, 240001)
    from scipy.stats import norm
    assert np.abs(O.gelu_tanh(w) - w * norm.cdf(w)).max() < 4.74e-4


def check_layernorm_hand():
    eps = 1e-5
    # row [3, 1]: mean 2, biased variance 1  ->  +-1/sqrt(1+eps)
    y = O.layernorm(np.array([[3.0, 1.0]]), eps=eps)
    np.testing.assert_allclose(y, [[1 / math.sqrt(1 + eps), -1 / math.sqrt(1 + eps)]], rtol=1e-15)
    # row [1,2,3,4]: mean 2.5, biased variance 1.25
    y = O.layernorm(np.array([[1.0, 2.0, 3.0, 4.0]]), eps=eps)
    np.testing.assert_allclose(y[0], (np.array([1, 2, 3, 4]) - 2.5) / math.sqrt(1.25 + eps), rtol=1e-15)
    # gamma, beta enter as gamma*n + beta
    g = np.array([2.0, -1.0, 0.5, 3.0])
    b = np.array([0.25, 1.0, -2.0, 0.0])
    y2 = O.layernorm(np.array([[1.0, 2.0, 3.0, 4.0]]), g, b, eps=eps)
    np.testing.assert_allclose(y2[0], y[0] * g + b, rtol=1e-15)


def check_layernorm_invariants():
    rng = np.random.default_rng(3)
    Z = rng.normal(1.5, 3.0, size=(17, 333))
    eps = 1e-5
    Y = O.layernorm(Z, eps=eps)
    np.testing.assert_allclose(Y.mean(axis=1), 0.0, atol=1e-12)
    s2 = np.var(Z, axis=1)  # ddof=0: the biased variance
    np.testing.assert_allclose(np.var(Y, axis=1), s2 / (s2 + eps), rtol=1e-12)


def check_mlp_exact_bruteforce():
    S, H, F = 3, 4, 6
    X, A, B = _small_int_case(11, S, H, F)
    Xf, Af, Bf = _to_frac(X), _to_frac(A), _to_frac(B)
    for act in ("relu", "none"):
        U = _exact_matmul(Xf, Af)
        G = _relu_frac(U) if act == "relu" else U
        V = _exact_matmul(G, Bf)
        Z = np.array([[float(Xf[i][j] + V[i][j]) for j in range(H)] for i in range(S)])
        got = O.mlp_block(X, A, B, act=act)
        np.testing.assert_allclose(got, O.layernorm(Z), rtol=0, atol=1e-12)


def check_mlp_closed_forms():
    rng = np.random.default_rng(5)
    X = rng.normal(size=(9, 16))
    I = np.eye(16)
    # A = B = I, no activation: Y = LN(2X)
    np.testing.assert_allclose(O.mlp_block(X, I, I, act="none"), O.layernorm(2 * X), atol=1e-12)
    # ReLU of an all-negative X A: Y = LN(X)
    Xp = np.abs(X) + 0.1
    An = -np.abs(rng.normal(size=(16, 24))) - 0.1
    Bn = rng.normal(size=(24, 16))
    np.testing.assert_allclose(O.mlp_block(Xp, An, Bn, act="relu"), O.layernorm(Xp), atol=1e-12)


def check_mlp_block_identities():
    inp = synth.gen_mlp(16, 32, 64, seed=2, dtype=torch.float32)
    ref = O.mlp_block(inp.X, inp.A, inp.B)
    for t in (1, 2, 4, 8):
        got = O.mlp_block_sharded(inp.X, synth.split_columns(inp.A, t), synth.split_rows(inp.B, t))
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # concat_i(X A_i) == X A  and  sum_i X_i B_i == X B
    A64 = inp.A.double().numpy()
    X64 = inp.X.double().numpy()
    cat = np.concatenate([O.linear_column(X64, Ai.double().numpy()) for Ai in synth.split_columns(inp.A, 4)], 1)
    np.testing.assert_allclose(cat, O.linear_column(X64, A64), atol=1e-12)
    Xs = np.split(X64, 4, axis=1)
    Bs = synth.split_rows(inp.A, 4)
    tot = sum(O.linear_row(Xi, Bi.double().numpy()) for Xi, Bi in zip(Xs, Bs))
    np.testing.assert_allclose(tot, O.linear_row(X64, A64), atol=1e-12)


def check_mlp_symmetries():
    inp = synth.gen_mlp(12, 16, 40, seed=9, dtype=torch.float32)
    Y = O.mlp_block(inp.X, inp.A, inp.B)
    rng = np.random.default_rng(1)
    p = rng.permutation(12)
    np.testing.assert_allclose(O.mlp_block(inp.X[p], inp.A, inp.B), Y[p], atol=1e-12)
    q = rng.permutation(40)
    np.testing.assert_allclose(O.mlp_block(inp.X, inp.A[:, q], inp.B[q, :]), Y, atol=1e-12)
    rows = [0, 5, 11]
    np.testing.assert_allclose(O.mlp_block(inp.X, inp.A, inp.B, rows=rows), Y[rows], atol=0)


def check_linears_exact():
    X, W, _ = _small_int_case(21, 5, 7, 3)
    ref = np.array(_exact_matmul(_to_frac(X), _to_frac(W)), dtype=np.float64)
    np.testing.assert_array_equal(O.linear_column(X, W), ref)
    np.testing.assert_array_equal(O.linear_row(X, W), ref)
    np.testing.assert_array_equal(O.linear_column(X, W, act="relu"), np.maximum(ref, 0))


def check_column_blocking():
    """The oracle forms wide products one block of output columns at a time.
    With a block of a few columns every product in the exact brute-force,
    closed-form and library pins crosses several blocks and ends in a ragged
    one, so a slice error in the block loop shows up against values computed
    without it."""
    saved = O._COL_BLOCK
    try:
        for blk in (1, 2, 3, 5):
            O._COL_BLOCK = blk
            check_mlp_exact_bruteforce()
            check_linears_exact()
            check_mlp_closed_forms()
            check_attention_library()
    finally:
        O._COL_BLOCK = saved


def check_attention_hand():
    # one head, d = 1, two keys: scores [0, ln 3] -> softmax [1/4, 3/4]
    Q = np.array([[1.0]])
    K = np.array([[0.0], [math.log(3.0)]])
    V = np.array([[4.0], [8.0]])
    np.testing.assert_allclose(O.attention_heads(Q, K, V, 1, 1), [[7.0]], rtol=1e-15)
    # d = 4 scales by 1/2: q.k = 2 ln 3 -> scaled ln 3 -> same weights
    Q4 = np.array([[1.0, 1.0, 0.0, 0.0]])
    K4 = np.array([[0.0] * 4, [math.log(3.0), math.log(3.0), 0.0, 0.0]])
    V4 = np.array([[4.0, 0, 0, 1], [8.0, 0, 0, 1]])
    np.testing.assert_allclose(O.attention_heads(Q4, K4, V4, 1, 4), [[7.0, 0, 0, 1]], rtol=1e-15)


def check_attention_uniform_keys():
    rng = np.random.default_rng(4)
    S, nh, d = 10, 3, 4
    Q = rng.normal(size=(S, nh * d))
    K = np.tile(rng.normal(size=(1, nh * d)), (S, 1))  # all key rows equal
    V = rng.normal(size=(S, nh * d))
    np.testing.assert_allclose(O.attention_heads(Q, K, V, nh, d),
                               np.tile(V.mean(axis=0), (S, 1)), atol=1e-13)


def check_attention_library():
    S, nh, d = 24, 4, 8
    H = nh * d
    inp = synth.gen_attn(S, H, seed=6, dtype=torch.float32)
    X = inp.X.double()
    Wqkv = inp.Wqkv.double()
    Wo = inp.Wo.double()
    # torch's multi-head attention keeps W in [out, in] layout: in_proj = Wqkv^T
    x = X.unsqueeze(1)  # [L, N=1, E]
    attn, _ = torch.nn.functional.multi_head_attention_forward(
        x, x, x, H, nh,
        in_proj_weight=Wqkv.T.contiguous(), in_proj_bias=torch.zeros(3 * H, dtype=torch.float64),
        bias_k=None, bias_v=None, add_zero_attn=False, dropout_p=0.0,
        out_proj_weight=Wo.T.contiguous(), out_proj_bias=torch.zeros(H, dtype=torch.float64),
        training=False, need_weights=False)
    Z = X.numpy() + attn.squeeze(1).numpy()
    ref = O.layernorm(Z)
    got = O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d)
    np.testing.assert_allclose(got, ref, atol=1e-11)
    rows = [0, 7, 23]
    np.testing.assert_allclose(O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d, rows=rows),
                               got[rows], atol=1e-12)
    # per head against torch's scaled-dot-product attention
    Q = X.numpy() @ Wqkv[:, :H].numpy()
    K = X.numpy() @ Wqkv[:, H:2 * H].numpy()
    Vv = X.numpy() @ Wqkv[:, 2 * H:].numpy()
    sd = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q).view(S, nh, d).transpose(0, 1),
        torch.from_numpy(K).view(S, nh, d).transpose(0, 1),
        torch.from_numpy(Vv).view(S, nh, d).transpose(0, 1))
    np.testing.assert_allclose(O.attention_heads(Q, K, Vv, nh, d),
                               sd.transpose(0, 1).reshape(S, H).numpy(), atol=1e-12)


def check_attention_row_equivariance():
    S, nh, d = 16, 2, 8
    inp = synth.gen_attn(S, nh * d, seed=8, dtype=torch.float32)
    Y = O.attention_sublayer(inp.X, inp.Wqkv, inp.Wo, nh, d)
    p = np.random.default_rng(2).permutation(S)
    np.testing.assert_allclose(O.attention_sublayer(inp.X[p], inp.Wqkv, inp.Wo, nh, d), Y[p], atol=1e-12)


def check_block_composition():
    S, nh, d, F = 16, 2, 8, 48
    H = nh * d
    a = synth.gen_attn(S, H, seed=12, dtype=torch.float32)
    m = synth.gen_mlp(S, H, F, seed=13, dtype=torch.float32)
    # post-LN block = the two pinned sublayers applied in turn
    Y1 = O.attention_sublayer(a.X, a.Wqkv, a.Wo, nh, d)
    ref = O.mlp_block(Y1, m.A, m.B)
    np.testing.assert_allclose(O.transformer_block(a.X, a.Wqkv, a.Wo, m.A, m.B, nh, d), ref, atol=1e-11)
    # zero output projections make the pre-LN block the identity on X ...
    Z = np.zeros_like(a.Wo.numpy())
    Zb = np.zeros_like(m.B.numpy())
    np.testing.assert_allclose(O.transformer_block(a.X, a.Wqkv, Z, m.A, Zb, nh, d, pre_ln=True),
                               a.X.double().numpy(), atol=0)
    # ... and the post-LN block LN(LN(X))
    np.testing.assert_allclose(O.transformer_block(a.X, a.Wqkv, Z, m.A, Zb, nh, d),
                               O.layernorm(O.layernorm(a.X.double().numpy())), atol=1e-12)
    # pre-LN: the MLP sees LN2 of the attention residual stream, the residual is unnormalised
    h1 = O.layernorm(a.X.double().numpy())
    Zr = a.X.double().numpy() + O.attention_out(h1, a.Wqkv, a.Wo, nh, d)
    pre = O.transformer_block(a.X, a.Wqkv, a.Wo, m.A, m.B, nh, d, pre_ln=True)
    np.testing.assert_allclose(pre, Zr + O.mlp_out(O.layernorm(Zr), m.A, m.B), atol=1e-11)
    # attention_out + residual + LN is the pinned attention sublayer
    np.testing.assert_allclose(O.layernorm(a.X.double().numpy() + O.attention_out(a.X, a.Wqkv, a.Wo, nh, d)), Y1,
                               atol=1e-12)
    rows = [1, 9, 15]
    np.testing.assert_allclose(O.transformer_block(a.X, a.Wqkv, a.Wo, m.A, m.B, nh, d, pre_ln=True, rows=rows),
                               pre[rows], atol=1e-12)


# ------------------------------------------------------------ backward pass

def _backward_case(S, H, F, seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((S, H))
    A = rng.standard_normal((H, F)) / math.sqrt(H)
    B = rng.standard_normal((F, H)) / math.sqrt(F)
    g = 1.0 + 0.5 * rng.standard_normal(H)
    b = 0.3 * rng.standard_normal(H)
    dY = rng.standard_normal((S, H))
    return X, A, B, g, b, dY


def check_backward_finite_differences():
    """Brute force: every gradient entry against a central difference of the
    (separately pinned) forward, L = sum(dY * Y), on a tiny rectangular case."""
    S, H, F = 3, 5, 7
    h = 1e-5
    for act in ("gelu_tanh", "gelu_erf", "relu", "none"):
        X, A, B, g, b, dY = _backward_case(S, H, F, seed=len(act))
        assert np.abs(X @ A).min() > 1e-3  # keep ReLU away from its kink
        grads = O.mlp_block_backward(X, A, B, dY, g, b, act=act)
        params = {"dX": X, "dA": A, "dB": B, "dgamma": g, "dbeta": b}

        def loss():
            return float((dY * O.mlp_block(X, A, B, g, b, act=act)).sum())

        for key, P in params.items():
            assert grads[key].shape == P.shape, key
            for idx in np.ndindex(*P.shape):
                old = P[idx]
                P[idx] = old + h
                lp = loss()
                P[idx] = old - h
                lm = loss()
                P[idx] = old
                fd = (lp - lm) / (2 * h)
                assert abs(fd - grads[key][idx]) <= 1e-7 * max(1.0, abs(fd)), (act, key, idx, fd, grads[key][idx])


def check_backward_autograd():
    """Library route: torch autograd (fp64) through torch's own layer_norm and
    GeLU/ReLU gives the same gradients."""
    S, H, F = 6, 8, 12
    fns = {"gelu_tanh": lambda u: torch.nn.functional.gelu(u, approximate="tanh"),
           "gelu_erf": lambda u: torch.nn.functional.gelu(u), "relu": torch.relu, "none": lambda u: u}
    for act, fn in fns.items():
        X, A, B, g, b, dY = _backward_case(S, H, F, seed=7 + len(act))
        ts = [torch.tensor(v, dtype=torch.float64, requires_grad=True) for v in (X, A, B, g, b)]
        Xt, At, Bt, gt, bt = ts
        Y = torch.nn.functional.layer_norm(Xt + fn(Xt @ At) @ Bt, (H,), gt, bt, eps=1e-5)
        (Y * torch.tensor(dY)).sum().backward()
        ref = O.mlp_block_backward(X, A, B, dY, g, b, act=act)
        for key, t in zip(("dX", "dA", "dB", "dgamma", "dbeta"), ts):
            np.testing.assert_allclose(ref[key], t.grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=f"{act} {key}")


def check_backward_invariants():
    """LayerNorm's input gradient has zero row sums (shifting a row does not
    change its normalisation); gamma = 0 blocks every gradient but dbeta's and
    dgamma's; the shard-by-shard form (weight gradients split like the weights,
    dX summed over the row split) equals the unsplit one."""
    X, A, B, g, b, dY = _backward_case(5, 8, 16, seed=3)
    Z = X + O.gelu_tanh(X @ A) @ B
    dZ, dg, db = O.layernorm_backward(Z, dY, g)
    np.testing.assert_allclose(dZ.sum(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose(db, dY.sum(axis=0), atol=1e-12)
    z = O.mlp_block_backward(X, A, B, dY, np.zeros(8), b)
    for key in ("dX", "dA", "dB"):
        assert np.abs(z[key]).max() == 0.0, key
    full = O.mlp_block_backward(X, A, B, dY, g, b)
    t = 4
    dZ, _, _ = O.layernorm_backward(Z, dY, g)
    dX = dZ.copy()
    for Ai, Bi in zip(np.split(A, t, axis=1), np.split(B, t, axis=0)):
        Ui = X @ Ai
        dUi = (dZ @ Bi.T) * O.activation_grad(Ui, "gelu_tanh")
        dX += dUi @ Ai.T
    np.testing.assert_allclose(dX, full["dX"], atol=1e-12)
    for i, (Ai, Bi) in enumerate(zip(np.split(A, t, axis=1), np.split(B, t, axis=0))):
        Ui = X @ Ai
        dUi = (dZ @ Bi.T) * O.activation_grad(Ui, "gelu_tanh")
        np.testing.assert_allclose(X.T @ dUi, full["dA"][:, i * 4:(i + 1) * 4], atol=1e-12)
        np.testing.assert_allclose(O.gelu_tanh(Ui).T @ dZ, full["dB"][i * 4:(i + 1) * 4], atol=1e-12)


def _attn_backward_case(S, nh, d, seed):
    rng = np.random.default_rng(seed)
    H = nh * d
    X = rng.standard_normal((S, H))
    Wqkv = rng.standard_normal((H, 3 * H)) / math.sqrt(H)
    Wo = rng.standard_normal((H, H)) / math.sqrt(H)
    g = 1.0 + 0.5 * rng.standard_normal(H)
    b = 0.3 * rng.standard_normal(H)
    dY = rng.standard_normal((S, H))
    return X, Wqkv, Wo, g, b, dY


def check_attention_backward_finite_differences():
    """Brute force: every gradient entry of the attention sublayer against a
    central difference of the (separately pinned) forward, L = sum(dY * Y)."""
    S, nh, d = 4, 2, 3
    h = 1e-5
    X, Wqkv, Wo, g, b, dY = _attn_backward_case(S, nh, d, seed=21)
    grads = O.attention_sublayer_backward(X, Wqkv, Wo, nh, d, dY, g, b)
    params = {"dX": X, "dWqkv": Wqkv, "dWo": Wo, "dgamma": g, "dbeta": b}

    def loss():
        return float((dY * O.attention_sublayer(X, Wqkv, Wo, nh, d, g, b)).sum())

    for key, P in params.items():
        assert grads[key].shape == P.shape, key
        for idx in np.ndindex(*P.shape):
            old = P[idx]
            P[idx] = old + h
            lp = loss()
            P[idx] = old - h
            lm = loss()
            P[idx] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grads[key][idx]) <= 1e-7 * max(1.0, abs(fd)), (key, idx, fd, grads[key][idx])


def check_attention_backward_autograd():
    """Library route: torch autograd (fp64) through torch's multi-head attention
    functional and layer_norm gives the same gradients."""
    S, nh, d = 8, 2, 4
    H = nh * d
    X, Wqkv, Wo, g, b, dY = _attn_backward_case(S, nh, d, seed=22)
    ts = [torch.tensor(v, dtype=torch.float64, requires_grad=True) for v in (X, Wqkv, Wo, g, b)]
    Xt, Wt, Wot, gt, bt = ts
    x = Xt.unsqueeze(1)  # [S, batch 1, H]
    att, _ = torch.nn.functional.multi_head_attention_forward(
        x, x, x, H, nh, Wt.T.contiguous(), None, None, None, False, 0.0, Wot.T.contiguous(), None,
        training=False, need_weights=False)
    Y = torch.nn.functional.layer_norm(Xt + att.squeeze(1), (H,), gt, bt, eps=1e-5)
    (Y * torch.tensor(dY)).sum().backward()
    ref = O.attention_sublayer_backward(X, Wqkv, Wo, nh, d, dY, g, b)
    for key, t in zip(("dX", "dWqkv", "dWo", "dgamma", "dbeta"), ts):
        np.testing.assert_allclose(ref[key], t.grad.numpy(), rtol=1e-9, atol=1e-11, err_msg=key)


ALL_CHECKS = [
    check_gelu_library, check_gelu_identities, check_layernorm_hand, check_layernorm_invariants,
    check_mlp_exact_bruteforce, check_mlp_closed_forms, check_mlp_block_identities,
    check_mlp_symmetries, check_linears_exact, check_column_blocking, check_attention_hand,
    check_attention_uniform_keys, check_attention_library, check_attention_row_equivariance,
    check_block_composition, check_backward_finite_differences, check_backward_autograd,
    check_backward_invariants, check_attention_backward_finite_differences, check_attention_backward_autograd,
]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check()


# -------------------------------------------------------- planted mistakes

def _fails_some_pin():
    for c in ALL_CHECKS:
        try:
            c()
        except AssertionError:
            return True
    return False


def _bad_layernorm_unbiased(Z, gamma=None, beta=None, eps=1e-5):
    Z = np.asarray(Z, dtype=np.float64)
    H = Z.shape[-1]
    mean = Z.mean(axis=-1, keepdims=True)
    var = ((Z - mean) ** 2).sum(axis=-1, keepdims=True) / (H - 1)
    Y = (Z - mean) / np.sqrt(var + eps)
    return Y * (1 if gamma is None else O._f64(gamma)) + (0 if beta is None else O._f64(beta))


def _bad_layernorm_eps_outside(Z, gamma=None, beta=None, eps=1e-5):
    Z = np.asarray(Z, dtype=np.float64)
    mean = Z.mean(axis=-1, keepdims=True)
    var = ((Z - mean) ** 2).mean(axis=-1, keepdims=True)
    Y = (Z - mean) / (np.sqrt(var) + eps)
    return Y * (1 if gamma is None else O._f64(gamma)) + (0 if beta is None else O._f64(beta))


def _bad_mlp_no_residual(X, A, B, gamma=None, beta=None, eps=1e-5, act="gelu_tanh", rows=None):
    Xr = O._rows(X, rows)
    return O.layernorm(O._matmul_cols(O._matmul_cols(Xr, A, act), B), gamma, beta, eps)


def _bad_mlp_act_after_b(X, A, B, gamma=None, beta=None, eps=1e-5, act="gelu_tanh", rows=None):
    Xr = O._rows(X, rows)
    return O.layernorm(Xr + O._matmul_cols(O._matmul_cols(Xr, A), B, act), gamma, beta, eps)


def _bad_gelu_constant(u):
    c = math.sqrt(2.0 / math.pi)
    return 0.5 * u * (1.0 + np.tanh(c * (u + 0.0447 * u ** 3)))


def _bad_gelu_no_half(u):
    return u * (1.0 + np.tanh(math.sqrt(2 / math.pi) * (u + 0.044715 * u ** 3))) / 1.999


def _bad_attention_no_scale(Q, K, V, nh, d):
    Oo = np.empty((Q.shape[0], nh * d))
    for h in range(nh):
        c = slice(h * d, (h + 1) * d)
        s = Q[:, c] @ K[:, c].T
        p = np.exp(s - s.max(axis=1, keepdims=True))
        Oo[:, c] = (p / p.sum(axis=1, keepdims=True)) @ V[:, c]
    return Oo


def _bad_attention_softmax_axis(Q, K, V, nh, d):
    Oo = np.empty((Q.shape[0], nh * d))
    for h in range(nh):
        c = slice(h * d, (h + 1) * d)
        s = Q[:, c] @ K[:, c].T / math.sqrt(d)
        p = np.exp(s - s.max(axis=0, keepdims=True))
        Oo[:, c] = (p / p.sum(axis=0, keepdims=True)) @ V[:, c]
    return Oo


def _bad_attention_wrong_head_cols(X, Wqkv, Wo, nh, d, gamma=None, beta=None, eps=1e-5, rows=None):
    # heads interleaved instead of contiguous d-column blocks
    X64 = O._f64(X)
    H = X64.shape[1]
    Xr = X64 if rows is None else X64[np.asarray(rows)]
    perm = np.arange(H).reshape(d, nh).T.reshape(-1)
    W = O._f64(Wqkv)
    Q = Xr @ W[:, :H][:, perm]
    K = X64 @ W[:, H:2 * H][:, perm]
    V = X64 @ W[:, 2 * H:][:, perm]
    Oo = O.attention_heads(Q, K, V, nh, d)[:, np.argsort(perm)]
    return O.layernorm(Xr + Oo @ O._f64(Wo), gamma, beta, eps)


def _bad_layernorm_backward_no_projection(Z, dY, gamma=None, eps=1e-5):
    Z = np.asarray(Z, dtype=np.float64)
    dY = O._f64(dY)
    H = Z.shape[-1]
    D = Z - Z.mean(axis=-1, keepdims=True)
    r = 1.0 / np.sqrt((D * D).mean(axis=-1, keepdims=True) + eps)
    g = dY * O._f64(gamma) if gamma is not None else dY
    return r * (g - g.sum(axis=-1, keepdims=True) / H), (dY * D * r).sum(axis=0), dY.sum(axis=0)


def _bad_activation_grad_is_activation(u, act):
    return O.activation(u, act)


def _bad_backward_no_residual(X, A, B, dY, gamma=None, beta=None, eps=1e-5, act="gelu_tanh"):
    X64, A64, B64 = O._f64(X), O._f64(A), O._f64(B)
    U = X64 @ A64
    G = O.activation(U, act)
    dZ, dg, db = O.layernorm_backward(X64 + G @ B64, dY, gamma, eps)
    dU = (dZ @ B64.T) * O.activation_grad(U, act)
    return {"dX": dU @ A64.T, "dA": X64.T @ dU, "dB": G.T @ dZ, "dgamma": dg, "dbeta": db}


def _bad_backward_db_from_u(X, A, B, dY, gamma=None, beta=None, eps=1e-5, act="gelu_tanh"):
    X64, A64, B64 = O._f64(X), O._f64(A), O._f64(B)
    U = X64 @ A64
    G = O.activation(U, act)
    dZ, dg, db = O.layernorm_backward(X64 + G @ B64, dY, gamma, eps)
    dU = (dZ @ B64.T) * O.activation_grad(U, act)
    return {"dX": dZ + dU @ A64.T, "dA": X64.T @ dU, "dB": U.T @ dZ, "dgamma": dg, "dbeta": db}


def _attention_backward_with(mistake: str):
    """The attention sublayer's chain rule with one plausible mistake in it."""
    def bad(X, Wqkv, Wo, nh, d, dY, gamma=None, beta=None, eps=1e-5):
        X64, W, Wo64 = O._f64(X), O._f64(Wqkv), O._f64(Wo)
        H = X64.shape[1]
        QKV = X64 @ W
        Q, K, V = QKV[:, :H], QKV[:, H:2 * H], QKV[:, 2 * H:]
        sc = 1.0 / math.sqrt(d)
        Oo = np.empty_like(Q)
        Ps = []
        for hh in range(nh):
            c = slice(hh * d, (hh + 1) * d)
            s_ = Q[:, c] @ K[:, c].T * sc
            p = np.exp(s_ - s_.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            Ps.append(p)
            Oo[:, c] = p @ V[:, c]
        dZ, dg, db = O.layernorm_backward(X64 + Oo @ Wo64, dY, gamma, eps)
        dO = dZ @ Wo64.T
        dQKV = np.empty_like(QKV)
        for hh in range(nh):
            c = slice(hh * d, (hh + 1) * d)
            p = Ps[hh]
            dP = dO[:, c] @ V[:, c].T
            if mistake == "no_softmax_projection":
                dS = p * dP * sc
            else:
                dS = p * (dP - (p * dP).sum(axis=1, keepdims=True))
                if mistake != "no_scale":
                    dS = dS * sc
            dQKV[:, c] = dS @ K[:, c]
            dQKV[:, H + hh * d:H + (hh + 1) * d] = (dS if mistake == "dk_untransposed" else dS.T) @ Q[:, c]
            dQKV[:, 2 * H + hh * d:2 * H + (hh + 1) * d] = (p if mistake == "dv_untransposed" else p.T) @ dO[:, c]
        dX = dQKV @ W.T if mistake == "no_residual" else dZ + dQKV @ W.T
        dWo = dZ.T @ Oo if mistake == "dwo_transposed" else Oo.T @ dZ
        return {"dX": dX, "dWqkv": X64.T @ dQKV, "dWo": dWo, "dgamma": dg, "dbeta": db}
    bad.__name__ = f"_bad_attention_backward_{mistake}"
    return bad


def _bad_matmul_cols_short_block(Xr, W, act="none"):
    # each block stops one column short of the next block's start
    n = W.shape[1]
    out = np.zeros((Xr.shape[0], n), dtype=np.float64)
    for c0 in range(0, n, O._COL_BLOCK):
        c1 = min(n, c0 + O._COL_BLOCK - 1)
        out[:, c0:c1] = O.activation(Xr @ O._f64(W[:, c0:c1]), act)
    return out


def _bad_matmul_cols_ragged_tail_dropped(Xr, W, act="none"):
    # the last, partial block is never formed
    n = W.shape[1]
    out = np.zeros((Xr.shape[0], n), dtype=np.float64)
    for c0 in range(0, n - n % O._COL_BLOCK, O._COL_BLOCK):
        c1 = c0 + O._COL_BLOCK
        out[:, c0:c1] = O.activation(Xr @ O._f64(W[:, c0:c1]), act)
    return out


_PLANTED = [
    ("layernorm", _bad_layernorm_unbiased),
    ("layernorm", _bad_layernorm_eps_outside),
    ("mlp_block", _bad_mlp_no_residual),
    ("mlp_block", _bad_mlp_act_after_b),
    ("gelu_tanh", _bad_gelu_constant),
    ("gelu_tanh", _bad_gelu_no_half),
    ("attention_heads", _bad_attention_no_scale),
    ("attention_heads", _bad_attention_softmax_axis),
    ("attention_sublayer", _bad_attention_wrong_head_cols),
    ("layernorm_backward", _bad_layernorm_backward_no_projection),
    ("activation_grad", _bad_activation_grad_is_activation),
    ("mlp_block_backward", _bad_backward_no_residual),
    ("mlp_block_backward", _bad_backward_db_from_u),
    ("_matmul_cols", _bad_matmul_cols_short_block),
    ("_matmul_cols", _bad_matmul_cols_ragged_tail_dropped),
] + [("attention_sublayer_backward", _attention_backward_with(m))
      for m in ("no_softmax_projection", "no_scale", "dk_untransposed", "dv_untransposed", "dwo_transposed",
                "no_residual")]


@pytest.mark.parametrize("name,bad", _PLANTED, ids=lambda x: getattr(x, "__name__", x))
def test_planted_mistake_is_caught(monkeypatch, name, bad):
    monkeypatch.setattr(O, name, bad)
    if name == "gelu_tanh":
        monkeypatch.setitem(O._ACTS, "gelu_tanh", bad)
    assert _fails_some_pin(), f"planted mistake in {name} passed every pin"
