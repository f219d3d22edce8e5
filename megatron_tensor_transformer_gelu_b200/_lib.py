"""ctypes binding of libtpblock.so (argument marshalling only).

Every step of the sublayer runs in the library's CUDA kernels; this module
only turns torch tensors into pointers and sizes and maps status codes to
exceptions.  If the library is missing it raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtpblock.so")

TP_OK = 0
STATUS = {
    0: "TP_OK", 1: "TP_ERR_INVALID_ARG", 2: "TP_ERR_UNSUPPORTED_SHAPE",
    3: "TP_ERR_WORKSPACE_TOO_SMALL", 4: "TP_ERR_CUDA", 5: "TP_ERR_TIMEOUT", 6: "TP_ERR_NO_DEVICE",
}
DTYPE = {torch.float32: 0, torch.bfloat16: 1}
ACT = {"none": 0, "gelu_tanh": 1, "gelu_erf": 2, "relu": 3}
MAX_SHARDS = 8

# name -> (restype, argtypes)
_c_int, _c_size, _c_float, _vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p
_vpp = ctypes.POINTER(ctypes.c_void_p)
SIGNATURES = {
    "tp_version": (_c_int, []),
    "tp_status_string": (ctypes.c_char_p, [_c_int]),
    "tp_device_error": (_c_int, []),
    "tp_mlp_workspace_bytes": (_c_size, [_c_int] * 5),
    "tp_mlp_forward": (_c_int, [_c_int] * 6 + [_vp, _vpp, _vpp, _vp, _vp, _c_float, _c_int, _vp, _vp, _c_size, _vp]),
    "tp_noalloc_scratch_bytes": (_c_size, []),
    "tp_mlp_forward_noalloc": (_c_int, [_c_int] * 6 + [_vp, _vpp, _vpp, _vp, _vp, _c_float, _c_int, _vp, _vp]),
    "tp_attn_workspace_bytes": (_c_size, [_c_int] * 6),
    "tp_qkv_attn_oproj_forward": (_c_int, [_c_int] * 7 + [_vp, _vpp, _vpp, _vp, _vp, _c_float, _vp, _vp, _c_size, _vp]),
    "tp_block_workspace_bytes": (_c_size, [_c_int] * 7),
    "tp_transformer_block_forward": (_c_int, [_c_int] * 9 + [_vp, _vpp, _vpp, _vpp, _vpp, _vp, _vp, _vp, _vp, _c_float,
                                                              _c_int, _vp, _vp, _c_size, _vp]),
    "tp_transformer_block_forward_ex": (_c_int, [_c_int] * 10 + [_vp, _vpp, _vpp, _vpp, _vpp, _vp, _vp, _vp, _vp,
                                                                  _c_float, _c_int, _vp, _vp, _c_size, _vp]),
    "tp_linear_column_forward": (_c_int, [_c_int] * 6 + [_vp, _vpp, _c_int, _vp, _vp]),
    "tp_linear_column_forward_ex": (_c_int, [_c_int] * 7 + [_vp, _vpp, _c_int, _vp, _vp]),
    "tp_linear_row_forward_ex": (_c_int, [_c_int] * 7 + [_vp, _vpp, _vp, _vp, _c_size, _vp]),
    "tp_mlp_forward_ex": (_c_int, [_c_int] * 7 + [_vp, _vpp, _vpp, _vp, _vp, _c_float, _c_int, _vp, _vp, _c_size,
                                                   _vp]),
    "tp_qkv_attn_oproj_forward_ex": (_c_int, [_c_int] * 8 + [_vp, _vpp, _vpp, _vp, _vp, _c_float, _vp, _vp, _c_size,
                                                              _vp]),
    "tp_linear_row_forward": (_c_int, [_c_int] * 6 + [_vp, _vpp, _vp, _vp, _c_size, _vp]),
    "tp_reduce_residual_layernorm": (_c_int, [_c_int] * 3 + [_vp, _vp, _c_int, _vp, _vp, _c_float, _vp, _c_int, _vp]),
    "tp_mlp_train_state_bytes": (_c_size, [_c_int] * 5),
    "tp_mlp_forward_train": (_c_int, [_c_int] * 6 + [_vp, _vpp, _vpp, _vp, _vp, _c_float, _c_int, _vp, _vp, _c_size,
                                                      _vp]),
    "tp_mlp_forward_train_ex": (_c_int, [_c_int] * 7 + [_vp, _vpp, _vpp, _vp, _vp, _c_float, _c_int, _vp, _vp,
                                                         _c_size, _vp]),
    "tp_mlp_backward_ex": (_c_int, [_c_int] * 6 + [_vp, _vpp, _vpp, _vp, _c_float, _c_int, _vp, _c_size, _vp, _vp,
                                                    _vpp, _vpp, _vp, _vp, _vp, _c_size, _vp]),
    "tp_mlp_backward_workspace_bytes": (_c_size, [_c_int] * 5),
    "tp_mlp_backward": (_c_int, [_c_int] * 5 + [_vp, _vpp, _vpp, _vp, _c_float, _c_int, _vp, _c_size, _vp, _vp, _vpp,
                                                 _vpp, _vp, _vp, _vp, _c_size, _vp]),
    "tp_attn_train_state_bytes": (_c_size, [_c_int] * 6),
    "tp_attn_forward_train": (_c_int, [_c_int] * 7 + [_vp, _vpp, _vpp, _vp, _vp, _c_float, _vp, _vp, _c_size, _vp]),
    "tp_attn_backward_workspace_bytes": (_c_size, [_c_int] * 6),
    "tp_attn_backward": (_c_int, [_c_int] * 6 + [_vp, _vpp, _vpp, _vp, _c_float, _vp, _c_size, _vp, _vp, _vpp, _vpp,
                                                  _vp, _vp, _vp, _c_size, _vp]),
    "tp_mlp_partial_workspace_bytes": (_c_size, [_c_int] * 5),
    "tp_mlp_partial_forward": (_c_int, [_c_int] * 5 + [_vp, _vpp, _vpp, _c_int, _vp, _vp, _c_size, _vp]),
    "tp_attn_partial_workspace_bytes": (_c_size, [_c_int] * 6),
    "tp_attn_partial_forward": (_c_int, [_c_int] * 6 + [_vp, _vpp, _vpp, _vp, _vp, _c_size, _vp]),
    "tp_reduce_residual_layernorm_multi": (_c_int, [_c_int] * 3 + [_vpp, _vp, _c_int, _vp, _vp, _c_float, _c_int,
                                                                   _vpp, _c_int, _vp]),
    "tp_ipc_export": (_c_int, [_vp, _vp]),
    "tp_ipc_import": (_c_int, [_vp, ctypes.POINTER(_vp)]),
    "tp_ipc_close": (_c_int, [_vp]),
    "tp_peer_barrier": (_c_int, [_c_int, _c_int, _vpp, ctypes.c_ulonglong, _vp]),
    "tp_set_gemm_tile_n": (_c_int, [_c_int]),
    "tp_gemm_plan": (_c_int, [_c_int] * 10 + [ctypes.POINTER(_c_int), ctypes.POINTER(_c_int)]),
    "tp_set_gemm_stream_k": (_c_int, [_c_int]),
    "tp_set_attn_kv_split": (_c_int, [_c_int]),
    "tp_attn_split_plan": (_c_int, [_c_int] * 4 + [_c_size] + [ctypes.POINTER(_c_int)] * 3),
    "tp_gemm_plan_sk": (_c_int, [_c_int] * 10 + [_c_size] + [ctypes.POINTER(_c_int)] * 4),
    "tp_gemm_plan_ex": (_c_int, [_c_int] * 11 + [_c_size] + [ctypes.POINTER(_c_int)] * 4),
    "tp_selftest_wait_timeout": (_c_int, [ctypes.c_longlong, _vp]),
    "tp_selftest_flag_wait_timeout": (_c_int, [ctypes.c_longlong, _vp]),
    "tp_selftest_exp2": (_c_int, [_vp, _vp, _vp, _c_int, _vp]),
    "tp_selftest_exp2_form": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _vp]),
    "tp_profile_enable": (_c_int, [_c_int]),
    "tp_profile_sample": (_c_int, [_c_int]),
    "tp_profile_collect": (_c_int, [ctypes.POINTER(_c_int), ctypes.POINTER(_c_int), ctypes.POINTER(ctypes.c_double),
                                    _c_int]),
    "tp_kernel_kind_name": (ctypes.c_char_p, [_c_int]),
}

_lib = None


class TPError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libtpblock.so (built by ``build()``); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run megatron_tensor_transformer_gelu_b200.build")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _check(code: int, where: str):
    if code != TP_OK:
        raise TPError(code, where)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _ptrs(ts):
    arr = (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])
    return ctypes.cast(arr, _vpp), arr


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def mlp_workspace_bytes(S, H, F, t, dtype) -> int:
    return lib().tp_mlp_workspace_bytes(S, H, F, t, DTYPE[dtype])


def attn_workspace_bytes(S, H, nh, d, t, dtype=torch.bfloat16) -> int:
    return lib().tp_attn_workspace_bytes(S, H, nh, d, t, DTYPE[dtype])


LAYOUT = {"in_out": 0, "out_in": 1}


def mlp_forward(X, A_shards, B_shards, Y, workspace, gamma=None, beta=None, eps=1e-5,
                act="gelu_tanh", stream=None, layout="in_out"):
    """layout "in_out": A_i [H, F/t], B_i [F/t, H]; "out_in" (nn.Linear): A_i [F/t, H], B_i [H, F/t]."""
    S, H = X.shape
    t = len(A_shards)
    F = sum(a.shape[1 if layout == "in_out" else 0] for a in A_shards)
    pa, ka = _ptrs(A_shards)
    pb, kb = _ptrs(B_shards)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if layout == "in_out":
        code = lib().tp_mlp_forward(S, H, F, t, DTYPE[X.dtype], DTYPE[Y.dtype], _ptr(X), pa, pb,
                                    _ptr(gamma), _ptr(beta), float(eps), ACT[act], _ptr(Y),
                                    _ptr(workspace), ws_bytes, _stream(stream))
    else:
        code = lib().tp_mlp_forward_ex(S, H, F, t, DTYPE[X.dtype], DTYPE[Y.dtype], LAYOUT[layout], _ptr(X), pa, pb,
                                       _ptr(gamma), _ptr(beta), float(eps), ACT[act], _ptr(Y),
                                       _ptr(workspace), ws_bytes, _stream(stream))
    _check(code, "tp_mlp_forward")


def mlp_forward_noalloc(X, A_shards, B_shards, Y, gamma=None, beta=None, eps=1e-5, act="gelu_tanh",
                       stream=None):
    """tp_mlp_forward with the library's fixed scratch array instead of a workspace."""
    S, H = X.shape
    t = len(A_shards)
    F = sum(a.shape[1] for a in A_shards)
    pa, ka = _ptrs(A_shards)
    pb, kb = _ptrs(B_shards)
    code = lib().tp_mlp_forward_noalloc(S, H, F, t, DTYPE[X.dtype], DTYPE[Y.dtype], _ptr(X), pa, pb,
                                        _ptr(gamma), _ptr(beta), float(eps), ACT[act], _ptr(Y), _stream(stream))
    _check(code, "tp_mlp_forward_noalloc")


def attn_forward(X, Wqkv_shards, Wo_shards, nh, d, Y, workspace, gamma=None, beta=None, eps=1e-5,
                 stream=None, layout="in_out"):
    S, H = X.shape
    t = len(Wqkv_shards)
    pq, kq = _ptrs(Wqkv_shards)
    po, ko = _ptrs(Wo_shards)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    code = lib().tp_qkv_attn_oproj_forward_ex(S, H, nh, d, t, DTYPE[X.dtype], DTYPE[Y.dtype], LAYOUT[layout],
                                              _ptr(X), pq, po, _ptr(gamma), _ptr(beta), float(eps), _ptr(Y),
                                              _ptr(workspace), ws_bytes, _stream(stream))
    _check(code, "tp_qkv_attn_oproj_forward")


def block_workspace_bytes(S, H, F, nh, d, t, dtype=torch.bfloat16) -> int:
    return lib().tp_block_workspace_bytes(S, H, F, nh, d, t, DTYPE[dtype])


def block_forward(X, Wqkv_shards, Wo_shards, A_shards, B_shards, nh, d, Y, workspace, pre_ln=False,
                  ln1=(None, None), ln2=(None, None), eps=1e-5, act="gelu_tanh", stream=None, layout="in_out"):
    """Attention sublayer then MLP sublayer (post-LN, or pre-LN with pre_ln=True)."""
    S, H = X.shape
    t = len(Wqkv_shards)
    F = sum(a.shape[1 if layout == "in_out" else 0] for a in A_shards)
    pq, kq = _ptrs(Wqkv_shards)
    po, ko = _ptrs(Wo_shards)
    pa, ka = _ptrs(A_shards)
    pb, kb = _ptrs(B_shards)
    code = lib().tp_transformer_block_forward_ex(
        S, H, F, nh, d, t, DTYPE[X.dtype], DTYPE[Y.dtype], 1 if pre_ln else 0, LAYOUT[layout], _ptr(X), pq, po, pa, pb,
        _ptr(ln1[0]), _ptr(ln1[1]), _ptr(ln2[0]), _ptr(ln2[1]), float(eps), ACT[act], _ptr(Y), _ptr(workspace),
        workspace.numel() * workspace.element_size() if workspace is not None else 0, _stream(stream))
    _check(code, "tp_transformer_block_forward")


def linear_column_forward(X, W_shards, Y, act="none", stream=None, layout="in_out"):
    M, K = X.shape
    t = len(W_shards)
    N = sum(w.shape[1 if layout == "in_out" else 0] for w in W_shards)
    pw, kw = _ptrs(W_shards)
    code = lib().tp_linear_column_forward_ex(M, K, N, t, DTYPE[X.dtype], DTYPE[Y.dtype], LAYOUT[layout], _ptr(X), pw,
                                             ACT[act], _ptr(Y), _stream(stream))
    _check(code, "tp_linear_column_forward")


def linear_row_forward(X, W_shards, Y, stream=None, layout="in_out"):
    M, K = X.shape
    t = len(W_shards)
    N = W_shards[0].shape[1 if layout == "in_out" else 0]
    pw, kw = _ptrs(W_shards)
    code = lib().tp_linear_row_forward_ex(M, K, N, t, DTYPE[X.dtype], DTYPE[Y.dtype], LAYOUT[layout], _ptr(X), pw,
                                          _ptr(Y), None, 0, _stream(stream))
    _check(code, "tp_linear_row_forward")


def reduce_residual_layernorm(parts, X, Y, gamma=None, beta=None, eps=1e-5, stream=None):
    """parts: None or an f32 tensor [nparts, S, H] (contiguous)."""
    S, H = X.shape
    nparts = 0 if parts is None else parts.shape[0]
    code = lib().tp_reduce_residual_layernorm(S, H, nparts, _ptr(parts), _ptr(X), DTYPE[X.dtype], _ptr(gamma),
                                              _ptr(beta), float(eps), _ptr(Y), DTYPE[Y.dtype], _stream(stream))
    _check(code, "tp_reduce_residual_layernorm")


def _addr(x) -> int:
    """Device address of a tensor, or an address given as an int (for example
    another GPU's buffer opened through CUDA IPC)."""
    return int(x) if isinstance(x, int) else x.data_ptr()


def _addrs(xs):
    arr = (ctypes.c_void_p * max(1, len(xs)))(*[_addr(x) for x in xs])
    return ctypes.cast(arr, _vpp), arr


IPC_HANDLE_BYTES = 72


def ipc_export(t) -> bytes:
    """CUDA IPC handle of a device tensor's allocation (to send to another rank's process)."""
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    _check(lib().tp_ipc_export(ctypes.c_void_p(t.data_ptr()), buf), "tp_ipc_export")
    return buf.raw


def ipc_import(handle: bytes) -> int:
    """Device address, on the current device, of another process's exported allocation."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("bad IPC handle")
    out = ctypes.c_void_p(0)
    buf = ctypes.create_string_buffer(bytes(handle), IPC_HANDLE_BYTES)
    _check(lib().tp_ipc_import(buf, ctypes.byref(out)), "tp_ipc_import")
    return int(out.value)


def ipc_close(addr: int) -> None:
    _check(lib().tp_ipc_close(ctypes.c_void_p(addr)), "tp_ipc_close")


def peer_barrier(nranks: int, rank: int, flag_arrays, epoch: int, stream=None) -> None:
    """flag_arrays: rank q's flag array (tensor or device address) for every q."""
    pf, kf = _addrs(flag_arrays)
    _check(lib().tp_peer_barrier(int(nranks), int(rank), pf, ctypes.c_ulonglong(int(epoch)), _stream(stream)),
           "tp_peer_barrier")


def mlp_partial_workspace_bytes(S, H, F, t, dtype=torch.bfloat16) -> int:
    return int(lib().tp_mlp_partial_workspace_bytes(S, H, F, t, DTYPE[dtype]))


def mlp_partial_forward(X, A_shards, B_shards, P, workspace, act="gelu_tanh", stream=None):
    """One rank's partial sum P = sum_i Act(X A_i) B_i (f32 [S, H]) over its shards."""
    S, H = X.shape
    t = len(A_shards)
    F = sum(a.shape[1] for a in A_shards)
    pa, ka = _ptrs(A_shards)
    pb, kb = _ptrs(B_shards)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    code = lib().tp_mlp_partial_forward(S, H, F, t, DTYPE[X.dtype], _ptr(X), pa, pb, ACT[act], _ptr(P),
                                        _ptr(workspace), ws_bytes, _stream(stream))
    _check(code, "tp_mlp_partial_forward")


def attn_partial_workspace_bytes(S, H, nh, d, t, dtype=torch.bfloat16) -> int:
    return int(lib().tp_attn_partial_workspace_bytes(S, H, nh, d, t, DTYPE[dtype]))


def attn_partial_forward(X, Wqkv_shards, Wo_shards, nh, d, P, workspace, stream=None):
    """One rank's partial sum P = sum_s O_s Wo_s (f32 [S, H]) over the nh heads its shards hold."""
    S, H = X.shape
    t = len(Wqkv_shards)
    pq, kq = _ptrs(Wqkv_shards)
    po, ko = _ptrs(Wo_shards)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    code = lib().tp_attn_partial_forward(S, H, nh, d, t, DTYPE[X.dtype], _ptr(X), pq, po, _ptr(P), _ptr(workspace),
                                         ws_bytes, _stream(stream))
    _check(code, "tp_attn_partial_forward")


def reduce_residual_layernorm_multi(rows, H, parts, X, Y_outs, x_dtype, out_dtype, gamma=None, beta=None, eps=1e-5,
                                    stream=None):
    """Y = LN(X + sum of the partials) for `rows` rows, into every output.
    parts, X, Y_outs: tensors or device addresses, each at the first of the rows."""
    pp, kp = _addrs(parts)
    py, ky = _addrs(Y_outs)
    code = lib().tp_reduce_residual_layernorm_multi(int(rows), int(H), len(parts), pp, ctypes.c_void_p(_addr(X)),
                                                    DTYPE[x_dtype], _ptr(gamma), _ptr(beta), float(eps),
                                                    len(Y_outs), py, DTYPE[out_dtype], _stream(stream))
    _check(code, "tp_reduce_residual_layernorm_multi")


def mlp_train_state_bytes(S, H, F, t, dtype=torch.bfloat16) -> int:
    return int(lib().tp_mlp_train_state_bytes(S, H, F, t, DTYPE[dtype]))


def mlp_backward_workspace_bytes(S, H, F, t, dtype=torch.bfloat16) -> int:
    return int(lib().tp_mlp_backward_workspace_bytes(S, H, F, t, DTYPE[dtype]))


def mlp_forward_train(X, A_shards, B_shards, Y, state, gamma=None, beta=None, eps=1e-5, act="gelu_tanh",
                      stream=None, layout="in_out"):
    S, H = X.shape
    t = len(A_shards)
    F = sum(a.shape[1 if layout == "in_out" else 0] for a in A_shards)
    pa, ka = _ptrs(A_shards)
    pb, kb = _ptrs(B_shards)
    code = lib().tp_mlp_forward_train_ex(S, H, F, t, DTYPE[X.dtype], DTYPE[Y.dtype], LAYOUT[layout], _ptr(X), pa, pb,
                                         _ptr(gamma), _ptr(beta), float(eps), ACT[act], _ptr(Y), _ptr(state),
                                         state.numel() * state.element_size(), _stream(stream))
    _check(code, "tp_mlp_forward_train")


def mlp_backward(X, A_shards, B_shards, state, dY, dX, dA_shards, dB_shards, workspace, gamma=None, dgamma=None,
                 dbeta=None, eps=1e-5, act="gelu_tanh", stream=None, layout="in_out"):
    """Gradients of one tp_mlp_forward_train call; dA/dB shards have the weights' layout."""
    S, H = X.shape
    t = len(A_shards)
    F = sum(a.shape[1 if layout == "in_out" else 0] for a in A_shards)
    pa, ka = _ptrs(A_shards)
    pb, kb = _ptrs(B_shards)
    pda, kda = _ptrs(dA_shards)
    pdb, kdb = _ptrs(dB_shards)
    code = lib().tp_mlp_backward_ex(S, H, F, t, DTYPE[X.dtype], LAYOUT[layout], _ptr(X), pa, pb, _ptr(gamma),
                                    float(eps), ACT[act], _ptr(state), state.numel() * state.element_size(),
                                    _ptr(dY), _ptr(dX), pda, pdb, _ptr(dgamma), _ptr(dbeta), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "tp_mlp_backward")


def attn_train_state_bytes(S, H, nh, d, t, dtype=torch.bfloat16) -> int:
    return int(lib().tp_attn_train_state_bytes(S, H, nh, d, t, DTYPE[dtype]))


def attn_backward_workspace_bytes(S, H, nh, d, t, dtype=torch.bfloat16) -> int:
    return int(lib().tp_attn_backward_workspace_bytes(S, H, nh, d, t, DTYPE[dtype]))


def attn_forward_train(X, Wqkv_shards, Wo_shards, nh, d, Y, state, gamma=None, beta=None, eps=1e-5, stream=None):
    S, H = X.shape
    t = len(Wqkv_shards)
    pq, kq = _ptrs(Wqkv_shards)
    po, ko = _ptrs(Wo_shards)
    code = lib().tp_attn_forward_train(S, H, nh, d, t, DTYPE[X.dtype], DTYPE[Y.dtype], _ptr(X), pq, po, _ptr(gamma),
                                       _ptr(beta), float(eps), _ptr(Y), _ptr(state),
                                       state.numel() * state.element_size(), _stream(stream))
    _check(code, "tp_attn_forward_train")


def attn_backward(X, Wqkv_shards, Wo_shards, nh, d, state, dY, dX, dWqkv_shards, dWo_shards, workspace, gamma=None,
                  dgamma=None, dbeta=None, eps=1e-5, stream=None):
    S, H = X.shape
    t = len(Wqkv_shards)
    pq, kq = _ptrs(Wqkv_shards)
    po, ko = _ptrs(Wo_shards)
    pdq, kdq = _ptrs(dWqkv_shards)
    pdo, kdo = _ptrs(dWo_shards)
    code = lib().tp_attn_backward(S, H, nh, d, t, DTYPE[X.dtype], _ptr(X), pq, po, _ptr(gamma), float(eps),
                                  _ptr(state), state.numel() * state.element_size(), _ptr(dY), _ptr(dX), pdq, pdo,
                                  _ptr(dgamma), _ptr(dbeta), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "tp_attn_backward")


def set_gemm_tile_n(tile_n: int) -> None:
    """0: the library's cost model picks GEMM tiles; 128: narrow tiles; 256..512:
    force that tile width."""
    _check(lib().tp_set_gemm_tile_n(int(tile_n)), "tp_set_gemm_tile_n")


def gemm_plan(M, t, row_mode, shard_k, shard_n, out_f32, b_kmajor=False, heavy_epilogue=False, slots=74,
              max_splits=1):
    """(tile_n, splits) the next GEMM launch of this shape would get (host logic only)."""
    tn, sp = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().tp_gemm_plan(int(M), int(t), int(bool(row_mode)), int(shard_k), int(shard_n), int(bool(out_f32)),
                              int(bool(b_kmajor)), int(bool(heavy_epilogue)), int(slots), int(max_splits),
                              ctypes.byref(tn), ctypes.byref(sp)), "tp_gemm_plan")
    return tn.value, sp.value


def set_gemm_stream_k(mode: int) -> None:
    """0: whole tiles only (the default); 1: stream-K wherever a launch has
    scratch for it; 2: the cost model decides per GEMM launch."""
    _check(lib().tp_set_gemm_stream_k(int(mode)), "tp_set_gemm_stream_k")


def gemm_plan_sk(M, t, row_mode, shard_k, shard_n, out_f32, b_kmajor=False, heavy_epilogue=False, slots=74,
                 max_splits=1, sk_area_bytes=0):
    """(tile_n, splits, stream_k, sk_clusters) of the next GEMM launch of this
    shape with sk_area_bytes of stream-K scratch (host logic only)."""
    out = [ctypes.c_int(0) for _ in range(4)]
    _check(lib().tp_gemm_plan_sk(int(M), int(t), int(bool(row_mode)), int(shard_k), int(shard_n),
                                 int(bool(out_f32)), int(bool(b_kmajor)), int(bool(heavy_epilogue)), int(slots),
                                 int(max_splits), int(sk_area_bytes), *[ctypes.byref(o) for o in out]),
           "tp_gemm_plan_sk")
    return tuple(o.value for o in out)


def set_attn_kv_split(mode: int) -> None:
    """Attention kernel's last-wave key split: 0 off, 1 the last partial wave
    (the default), 2 every unit."""
    _check(lib().tp_set_attn_kv_split(int(mode)), "tp_set_attn_kv_split")


def attn_split_plan(S, nh, slots=148, mode=1, scratch_bytes=1 << 40):
    """(whole, split, kv_half) of the attention kernel's key-split plan (host logic only)."""
    out = [ctypes.c_int(0) for _ in range(3)]
    _check(lib().tp_attn_split_plan(int(S), int(nh), int(slots), int(mode), int(scratch_bytes),
                                    *[ctypes.byref(o) for o in out]), "tp_attn_split_plan")
    return tuple(o.value for o in out)


def gemm_plan_ex(M, t, row_mode, shard_k, shard_n, out_f32, a_mnmajor=False, b_kmajor=False, heavy_epilogue=False,
                 slots=74, max_splits=1, sk_area_bytes=0):
    """gemm_plan_sk with A read M-major (the weight-gradient GEMMs) when a_mnmajor."""
    out = [ctypes.c_int(0) for _ in range(4)]
    _check(lib().tp_gemm_plan_ex(int(M), int(t), int(bool(row_mode)), int(shard_k), int(shard_n),
                                 int(bool(out_f32)), int(bool(a_mnmajor)), int(bool(b_kmajor)),
                                 int(bool(heavy_epilogue)), int(slots), int(max_splits), int(sk_area_bytes),
                                 *[ctypes.byref(o) for o in out]), "tp_gemm_plan_ex")
    return tuple(o.value for o in out)


def selftest_wait_timeout(limit_cycles: int, stream=None):
    _check(lib().tp_selftest_wait_timeout(int(limit_cycles), _stream(stream)), "tp_selftest_wait_timeout")


def selftest_flag_wait_timeout(limit_cycles: int, stream=None):
    _check(lib().tp_selftest_flag_wait_timeout(int(limit_cycles), _stream(stream)), "tp_selftest_flag_wait_timeout")


def selftest_exp2(x, stream=None, form=0):
    """(a polynomial 2^x, CUDA's exp2f(x)) for a device f32 tensor x: form 0
    the degree-4 single-value evaluation, form 1 the degree-3 pair (f32x2)
    evaluation the attention kernel's softmax uses."""
    yp = torch.empty_like(x)
    yr = torch.empty_like(x)
    _check(lib().tp_selftest_exp2_form(_ptr(x), _ptr(yp), _ptr(yr), x.numel(), int(form), _stream(stream)),
           "tp_selftest_exp2_form")
    return yp, yr


def device_error() -> int:
    return lib().tp_device_error()


def profile_enable(on: bool):
    _check(lib().tp_profile_enable(1 if on else 0), "tp_profile_enable")


def profile_sample(on: bool):
    _check(lib().tp_profile_sample(1 if on else 0), "tp_profile_sample")


def profile_collect(nkinds: int = 8):
    """{kernel kind: (launches, timed launches, summed ms of the timed ones)}"""
    launches = (ctypes.c_int * nkinds)()
    timed = (ctypes.c_int * nkinds)()
    ms = (ctypes.c_double * nkinds)()
    n = lib().tp_profile_collect(launches, timed, ms, nkinds)
    if n < 0:
        raise TPError(-n, "tp_profile_collect")
    return {lib().tp_kernel_kind_name(k).decode(): (launches[k], timed[k], ms[k]) for k in range(n)}
