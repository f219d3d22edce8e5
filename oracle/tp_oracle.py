"""fp64 CPU oracle of the tensor-parallel (Megatron) Transformer sublayer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may call it.  It shares no code with the CUDA path.

It computes the plain, unsharded definition of what the tensor-parallel split
computes exactly (up to rounding order).  Every input is the exact value the
GPU receives (bf16 or f32), widened to float64; every intermediate stays in
float64.  A matmul is done by numpy (a library primitive); nothing is blocked,
fused or reordered beyond the definition.  Where memory demands it, a product
is produced a block of *output columns* at a time, which leaves every output
element's own dot product unchanged.

Pages cited (by title and section):
  [TYPC]  "张量并行：千亿大模型突破单卡显存限制的底层技术" (typc.net)
  [0539]  "1. 张量并行：Tensor Parallelism" (0539edu.com news 288531)
  [PWWT]  "TP到底在切什么——从一次矩阵乘法说起" (pwwt.cn news 5934571)

Readings adopted where the pages are silent, garbled or contradict each other:
  * A is split by columns and B by rows ([TYPC] §3 MLP bullet; [0539] §1.2.1);
    the [PWWT] §2.3 labels are swapped and are not followed.
  * Post-LN: Y = LN(X + sum_i Act(X A_i) B_i); no LayerNorm on the input.
  * LayerNorm: biased variance (divide by H), eps inside the square root,
    Y = (Z - mean) / sqrt(var + eps) * gamma + beta.
  * GeLU: the tanh form 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)))
    (Hendrycks & Gimpel 2016); the erf form 0.5 u (1 + erf(u / sqrt 2)) and
    ReLU are the other activations ([0539] §1.2.1 names "ReLU or GeLU").
  * Attention: per head, softmax(Q K^T / sqrt(d)) V, non-causal, no mask,
    max-subtracted softmax; heads concatenated in head order, then O W_O.
  * No biases, no dropout.
  * Backward pass: the pages give no formulas, only that each shard computes
    the gradient of its own weight block ("TP到底在切什么" §4, weight
    gradients split like the weights) and that the two split directions
    differ in backward ("张量并行：千亿大模型突破单卡显存限制的底层技术" §2.2).
    The oracle is the gradient of the forward definition above by the chain
    rule, for a given upstream gradient dY (the vector-Jacobian product).

Parity status: every function below is pinned by tests/test_oracle_pins.py
(brute force on exact small inputs, closed forms, invariants, library
special cases); none is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "gelu_tanh", "gelu_erf", "relu", "activation",
    "layernorm", "mlp_block", "mlp_block_sharded",
    "linear_column", "linear_row",
    "attention_heads", "attention_sublayer", "attention_out", "mlp_out", "transformer_block",
    "activation_grad", "layernorm_backward", "mlp_block_backward", "attention_sublayer_backward",
]

_COL_BLOCK = 2048  # output-column block for products whose fp64 weight copy is large


def _f64(a) -> np.ndarray:
    """Exact widening of the GPU's input values (torch or numpy, bf16/f32) to fp64."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------- activations
# [0539] §1.2.1: Act is applied elementwise ("ReLU 或 GeLU"), so it can be
# applied to each column shard on its own.

def gelu_tanh(u: np.ndarray) -> np.ndarray:
    """tanh-approximated GeLU (Hendrycks & Gimpel 2016)."""
    c = math.sqrt(2.0 / math.pi)
    return 0.5 * u * (1.0 + np.tanh(c * (u + 0.044715 * u * u * u)))


def gelu_erf(u: np.ndarray) -> np.ndarray:
    """Exact GeLU, u * Phi(u) written through erf."""
    return 0.5 * u * (1.0 + _erf(u / math.sqrt(2.0)))


def relu(u: np.ndarray) -> np.ndarray:
    return np.maximum(u, 0.0)


_ACTS = {"none": lambda u: u, "gelu_tanh": gelu_tanh, "gelu_erf": gelu_erf, "relu": relu}


def activation(u: np.ndarray, act: str) -> np.ndarray:
    return _ACTS[act](u)


# ------------------------------------------------------------------ LayerNorm
# [PWWT] §2.3 and §5.3: the shard reduction is followed by the residual add and
# the next LayerNorm, whose row statistics are taken over the full hidden row.

def layernorm(Z: np.ndarray, gamma=None, beta=None, eps: float = 1e-5) -> np.ndarray:
    Z = np.asarray(Z, dtype=np.float64)
    H = Z.shape[-1]
    mean = Z.sum(axis=-1, keepdims=True) / H
    D = Z - mean
    var = (D * D).sum(axis=-1, keepdims=True) / H
    Y = D / np.sqrt(var + eps)
    if gamma is not None:
        Y = Y * _f64(gamma)
    if beta is not None:
        Y = Y + _f64(beta)
    return Y


# ------------------------------------------------------------------- products

def _matmul_cols(Xr: np.ndarray, W, act: str = "none") -> np.ndarray:
    """act(Xr @ W) with W widened to fp64 one block of output columns at a time."""
    n = W.shape[1]
    out = np.empty((Xr.shape[0], n), dtype=np.float64)
    for c0 in range(0, n, _COL_BLOCK):
        c1 = min(n, c0 + _COL_BLOCK)
        out[:, c0:c1] = activation(Xr @ _f64(W[:, c0:c1]), act)
    return out


def _rows(X, rows):
    X64 = _f64(X)
    return X64 if rows is None else X64[np.asarray(rows, dtype=np.int64)]


# ---------------------------------------------------------------------- MLP
# [0539] §1.2.1, eqs (1.2)-(1.5): Y_mlp = Act(X A) B.  Column-splitting A gives
# Act(X A) = [Act(X A_1) ... Act(X A_t)] ([TYPC] §2.1; [0539] §1.1 列切分), and
# row-splitting B gives [G_1 ... G_t] B = sum_i G_i B_i ([TYPC] §2.2; [0539]
# §1.1, eq (1.1) 外积和切分).  The oracle computes the unsplit left-hand sides.

def mlp_block(X, A, B, gamma=None, beta=None, eps: float = 1e-5,
              act: str = "gelu_tanh", rows=None) -> np.ndarray:
    """Y = LN(X + Act(X A) B) for the requested rows (all rows if None).

    Each output row depends only on the same row of X, so a row sample is
    exactly the corresponding rows of the full result."""
    Xr = _rows(X, rows)
    G = _matmul_cols(Xr, A, act)          # step 1-2: U = X A, G = Act(U)
    V = _matmul_cols(G, B)                # step 3:   V = G B
    Z = Xr + V                            # step 4:   residual
    return layernorm(Z, gamma, beta, eps)  # step 5:  LayerNorm


def mlp_block_sharded(X, A_shards, B_shards, gamma=None, beta=None, eps: float = 1e-5,
                      act: str = "gelu_tanh", rows=None) -> np.ndarray:
    """The split form sum_i Act(X A_i) B_i, shard by shard (self-tests only:
    it checks the block identities the method relies on)."""
    Xr = _rows(X, rows)
    acc = np.zeros((Xr.shape[0], _f64(B_shards[0]).shape[1]))
    for Ai, Bi in zip(A_shards, B_shards):
        acc += _f64(activation(Xr @ _f64(Ai), act)) @ _f64(Bi)
    return layernorm(Xr + acc, gamma, beta, eps)


# ------------------------------------------------------------ single linears
# [TYPC] §2.1 / [PWWT] §1.1 figure 1: the column-split linear concatenates
# X W_i, which equals X W.  [TYPC] §2.2 / [PWWT] §1.2 figure 2: the row-split
# linear sums X_i W_i (X split by columns, W by rows), which equals X W.

def linear_column(X, W, act: str = "none", rows=None) -> np.ndarray:
    return _matmul_cols(_rows(X, rows), W, act)


def linear_row(X, W, rows=None) -> np.ndarray:
    return _matmul_cols(_rows(X, rows), W)


# ---------------------------------------------------------------- attention
# [0539] §1.2.2 (eqs (1.6)-(1.13), formulas lost in extraction) and [PWWT]
# §2.2 figure 4: every head computes softmax(Q_h K_h^T / sqrt(d)) V_h on its own;
# the heads' outputs are concatenated and multiplied by W_O, which is why W_O
# is row-split by head ([0539] §1.2.2; [PWWT] §2.1 O 投影).

def attention_heads(Q: np.ndarray, K: np.ndarray, V: np.ndarray, nh: int, d: int) -> np.ndarray:
    """O = concat_h softmax(Q_h K_h^T / sqrt d) V_h; Q [r, nh*d], K, V [S, nh*d]."""
    O = np.empty((Q.shape[0], nh * d), dtype=np.float64)
    scale = 1.0 / math.sqrt(d)
    for h in range(nh):
        c = slice(h * d, (h + 1) * d)
        s = (Q[:, c] @ K[:, c].T) * scale
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        O[:, c] = p @ V[:, c]
    return O


def attention_out(Xin, Wqkv, Wo, nh: int, d: int, rows=None) -> np.ndarray:
    """concat_h(softmax(Q_h K_h^T / sqrt d) V_h) W_O for the requested query
    rows of the input Xin (no residual, no LayerNorm)."""
    X64 = _f64(Xin)
    H = X64.shape[1]
    assert nh * d == H
    Xr = X64 if rows is None else X64[np.asarray(rows, dtype=np.int64)]
    Q = _matmul_cols(Xr, Wqkv[:, 0:H])
    K = _matmul_cols(X64, Wqkv[:, H:2 * H])
    V = _matmul_cols(X64, Wqkv[:, 2 * H:3 * H])
    return _matmul_cols(attention_heads(Q, K, V, nh, d), Wo)


def mlp_out(Xin_rows, A, B, act: str = "gelu_tanh") -> np.ndarray:
    """Act(Xin A) B for the given input rows (no residual, no LayerNorm)."""
    return _matmul_cols(_matmul_cols(_f64(Xin_rows), A, act), B)


def transformer_block(X, Wqkv, Wo, A, B, nh: int, d: int, ln1=(None, None), ln2=(None, None),
                      eps: float = 1e-5, act: str = "gelu_tanh", pre_ln: bool = False, rows=None) -> np.ndarray:
    """One Transformer block: the attention sublayer then the MLP sublayer
    ("TP到底在切什么" §2.1 figure 3).  post-LN: Y1 = LN1(X + Attn(X)),
    Y = LN2(Y1 + MLP(Y1)).  pre-LN: Z1 = X + Attn(LN1(X)), Y = Z1 + MLP(LN2(Z1)).
    Every output row depends on all rows of X only through the attention's K
    and V, so a row sample is exact."""
    X64 = _f64(X)
    Xr = X64 if rows is None else X64[np.asarray(rows, dtype=np.int64)]
    if not pre_ln:
        Y1 = layernorm(Xr + attention_out(X64, Wqkv, Wo, nh, d, rows=rows), ln1[0], ln1[1], eps)
        return layernorm(Y1 + mlp_out(Y1, A, B, act), ln2[0], ln2[1], eps)
    h1 = layernorm(X64, ln1[0], ln1[1], eps)
    Z1 = Xr + attention_out(h1, Wqkv, Wo, nh, d, rows=rows)
    return Z1 + mlp_out(layernorm(Z1, ln2[0], ln2[1], eps), A, B, act)


def attention_sublayer(X, Wqkv, Wo, nh: int, d: int, gamma=None, beta=None,
                       eps: float = 1e-5, rows=None) -> np.ndarray:
    """Y = LN(X + concat_h(attn_h) W_O) for the requested query rows.

    Wqkv is [H, 3H] = [W_Q | W_K | W_V]; head h owns columns h*d..(h+1)*d-1 of
    each block.  K and V are needed for every row; Q only for the sampled rows."""
    X64 = _f64(X)
    H = X64.shape[1]
    assert nh * d == H
    Xr = X64 if rows is None else X64[np.asarray(rows, dtype=np.int64)]
    Q = _matmul_cols(Xr, Wqkv[:, 0:H])
    K = _matmul_cols(X64, Wqkv[:, H:2 * H])
    V = _matmul_cols(X64, Wqkv[:, 2 * H:3 * H])
    O = attention_heads(Q, K, V, nh, d)
    Z = Xr + _matmul_cols(O, Wo)
    return layernorm(Z, gamma, beta, eps)


# ------------------------------------------------------------- backward pass
# The gradient of the post-LN MLP sublayer for an upstream gradient dY, by the
# chain rule through the forward steps of mlp_block:
#   U = X A, G = Act(U), V = G B, Z = X + V, Y = LN(Z)
# Column-splitting A and row-splitting B split the weight gradients the same
# way ("TP到底在切什么" §4: each shard computes the gradient of its own block of
# W): dA = X^T dU gives dA_i = X^T dU_i (the columns of shard i), and
# dB = G^T dZ gives dB_i = G_i^T dZ (the rows of shard i); dX sums the row
# split's contributions, dX = dZ + sum_i dU_i A_i^T.

def activation_grad(u: np.ndarray, act: str) -> np.ndarray:
    """d Act(u) / du, elementwise.  ReLU's derivative at 0 is taken as 0."""
    if act == "gelu_tanh":
        c = math.sqrt(2.0 / math.pi)
        t = np.tanh(c * (u + 0.044715 * u * u * u))
        return 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * c * (1.0 + 3.0 * 0.044715 * u * u)
    if act == "gelu_erf":
        return 0.5 * (1.0 + _erf(u / math.sqrt(2.0))) + u * np.exp(-0.5 * u * u) / math.sqrt(2.0 * math.pi)
    if act == "relu":
        return (u > 0.0).astype(np.float64)
    if act == "none":
        return np.ones_like(u)
    raise KeyError(act)


def layernorm_backward(Z, dY, gamma=None, eps: float = 1e-5):
    """(dZ, dgamma, dbeta) of Y = (Z - mean) / sqrt(var + eps) * gamma + beta
    (biased variance over the last axis).  With xh the normalised row, r the
    reciprocal standard deviation and g = dY * gamma:
        dZ = r * (g - mean(g) - xh * mean(g * xh)),
        dgamma = sum over rows of dY * xh,  dbeta = sum over rows of dY."""
    Z = np.asarray(Z, dtype=np.float64)
    dY = _f64(dY)
    H = Z.shape[-1]
    mean = Z.sum(axis=-1, keepdims=True) / H
    D = Z - mean
    var = (D * D).sum(axis=-1, keepdims=True) / H
    r = 1.0 / np.sqrt(var + eps)
    xh = D * r
    g = dY * _f64(gamma) if gamma is not None else dY
    dZ = r * (g - g.sum(axis=-1, keepdims=True) / H - xh * ((g * xh).sum(axis=-1, keepdims=True) / H))
    return dZ, (dY * xh).sum(axis=0), dY.sum(axis=0)


def mlp_block_backward(X, A, B, dY, gamma=None, beta=None, eps: float = 1e-5,
                       act: str = "gelu_tanh") -> dict:
    """Gradients of mlp_block's output Y with respect to X, A, B, gamma and
    beta, contracted with dY: {"dX", "dA", "dB", "dgamma", "dbeta"}.  beta
    does not enter any gradient but its own (dbeta = column sums of dY)."""
    del beta
    X64 = _f64(X)
    A64 = _f64(A)
    B64 = _f64(B)
    U = X64 @ A64                          # forward, step 1
    G = activation(U, act)                 # step 2
    Z = X64 + G @ B64                      # steps 3-4
    dZ, dgamma, dbeta = layernorm_backward(Z, dY, gamma, eps)   # through step 5
    dG = dZ @ B64.T                        # through step 3 (V = G B)
    dU = dG * activation_grad(U, act)      # through step 2
    return {
        "dX": dZ + dU @ A64.T,             # residual path + through step 1
        "dA": X64.T @ dU,
        "dB": G.T @ dZ,
        "dgamma": dgamma,
        "dbeta": dbeta,
    }


# Backward of the post-LN attention sublayer for an upstream gradient dY, by
# the chain rule through attention_sublayer's steps:
#   Q, K, V = X W_Q, X W_K, X W_V;  per head h: S_h = Q_h K_h^T / sqrt(d),
#   P_h = softmax(S_h) (rows), O_h = P_h V_h;  Z = X + O W_O;  Y = LN(Z).
# The softmax backward of a row p with upstream g is p * (g - sum(g * p)).
# Splitting Wqkv by head and W_O by the matching rows splits their gradients
# the same way ("TP到底在切什么" §4): dWqkv = X^T dQKV, dW_O = O^T dZ.

def attention_sublayer_backward(X, Wqkv, Wo, nh: int, d: int, dY, gamma=None, beta=None,
                                eps: float = 1e-5) -> dict:
    """Gradients of attention_sublayer's output with respect to X, Wqkv, Wo,
    gamma and beta, contracted with dY: {"dX", "dWqkv", "dWo", "dgamma", "dbeta"}."""
    del beta
    X64 = _f64(X)
    W = _f64(Wqkv)
    Wo64 = _f64(Wo)
    H = X64.shape[1]
    assert nh * d == H
    QKV = X64 @ W
    Q, K, V = QKV[:, :H], QKV[:, H:2 * H], QKV[:, 2 * H:]
    scale = 1.0 / math.sqrt(d)
    O = np.empty_like(Q)
    P = []
    for h in range(nh):
        c = slice(h * d, (h + 1) * d)
        s = (Q[:, c] @ K[:, c].T) * scale
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        P.append(p)
        O[:, c] = p @ V[:, c]
    Z = X64 + O @ Wo64
    dZ, dgamma, dbeta = layernorm_backward(Z, dY, gamma, eps)
    dO = dZ @ Wo64.T
    dWo = O.T @ dZ
    dQKV = np.empty_like(QKV)
    for h in range(nh):
        c = slice(h * d, (h + 1) * d)
        p = P[h]
        dV = p.T @ dO[:, c]
        dP = dO[:, c] @ V[:, c].T
        dS = p * (dP - (dP * p).sum(axis=1, keepdims=True)) * scale
        dQKV[:, c] = dS @ K[:, c]
        dQKV[:, H + h * d:H + (h + 1) * d] = dS.T @ Q[:, c]
        dQKV[:, 2 * H + h * d:2 * H + (h + 1) * d] = dV
    return {
        "dX": dZ + dQKV @ W.T,
        "dWqkv": X64.T @ dQKV,
        "dWo": dWo,
        "dgamma": dgamma,
        "dbeta": dbeta,
    }
