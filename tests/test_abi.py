"""Host-only checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments before anything is launched.

No compute call is made here.  Argument checks run before any CUDA call, so
fake (aligned, never dereferenced) pointers are safe; the single case with
valid arguments is only run when no CUDA device is present, where it must
return TP_ERR_NO_DEVICE instead of launching.
"""
from __future__ import annotations

import ctypes
import os
import re

import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tpblock.h")

OK, INVALID, UNSUPPORTED, WS_SMALL, NO_DEVICE = 0, 1, 2, 3, 6
FAKE = 0x10000  # aligned, never dereferenced


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tp_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("tp_mlp_forward", "tp_qkv_attn_oproj_forward", "tp_linear_column_forward",
              "tp_linear_row_forward", "tp_reduce_residual_layernorm", "tp_mlp_workspace_bytes",
              "tp_attn_workspace_bytes", "tp_status_string", "tp_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
        assert n in L.SIGNATURES, f"binding lacks {n}"


def test_exports_only_c_symbols():
    out = os.popen(f"nm -D --defined-only {L.LIB_PATH}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    tp_syms = {s for s in exported if s.startswith("tp_")}
    assert tp_syms == set(declared_functions())


def test_version_and_status_strings(lib):
    assert lib.tp_version() == 1
    assert lib.tp_status_string(0) == b"ok"
    assert lib.tp_status_string(3) == b"workspace too small"
    assert lib.tp_status_string(99) == b"unknown status"


def test_workspace_sizes(lib):
    S, H, F = 2048, 4096, 16384
    assert lib.tp_mlp_workspace_bytes(S, H, F, 4, 1) == S * F * 2 + 4 * S * H * 4
    assert lib.tp_mlp_workspace_bytes(S, H, F, 4, 0) == S * F * 4 + 4 * S * H * 4
    assert lib.tp_mlp_workspace_bytes(-1, H, F, 4, 1) == 0
    assert lib.tp_attn_workspace_bytes(2048, 8192, 64, 128, 4, 1) == 2048 * 8192 * (6 + 2 + 16)
    assert lib.tp_attn_workspace_bytes(2048, 8192, 64, 128, 4, 0) == 0


def test_attention_backward_workspace(lib):
    """dZ, dO, dQKV (bf16), the f32 row-split partial, D [nh, S] and 640
    per-CTA LayerNorm partial rows; the fused attention backward keeps P and
    dS on chip, so no [S, S] matrix is held."""
    def expect(S, H, nh, g):
        return S * H * (2 + 2 + 6 + 4) + nh * S * 4 + 640 * 2 * H * 4
    lib.tp_attn_backward_workspace_bytes.restype = ctypes.c_size_t
    assert lib.tp_attn_backward_workspace_bytes(2048, 8192, 64, 128, 4, 1) == expect(2048, 8192, 64, 8)
    assert lib.tp_attn_backward_workspace_bytes(256, 512, 4, 128, 2, 1) == expect(256, 512, 4, 4)
    assert lib.tp_attn_backward_workspace_bytes(5888, 1024, 8, 128, 2, 1) == expect(5888, 1024, 8, 7)
    assert lib.tp_attn_backward_workspace_bytes(8192, 8192, 64, 128, 4, 1) == expect(8192, 8192, 64, 4)
    assert lib.tp_attn_backward_workspace_bytes(2048, 8192, 64, 128, 4, 0) == 0


def _ptrs(n, base=FAKE):
    arr = (ctypes.c_void_p * n)(*[base + 256 * i for i in range(n)])
    return ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)), arr


def _mlp(lib, S=128, H=256, F=1024, t=2, dtype=1, out=1, X=FAKE, A=None, Bp=None, eps=1e-5, act=1,
         Y=FAKE, ws=FAKE, ws_bytes=1 << 30):
    pa, ka = A if A is not None else _ptrs(t)
    pb, kb = Bp if Bp is not None else _ptrs(t)
    return lib.tp_mlp_forward(S, H, F, t, dtype, out, ctypes.c_void_p(X), pa, pb, None, None, eps, act,
                              ctypes.c_void_p(Y), ctypes.c_void_p(ws), ws_bytes, None)


def test_mlp_argument_checks(lib):
    assert _mlp(lib, t=0) == INVALID
    assert _mlp(lib, t=9) == INVALID
    assert _mlp(lib, X=0) == INVALID
    assert _mlp(lib, X=FAKE + 4) == INVALID            # misaligned
    assert _mlp(lib, Y=FAKE + 8) == INVALID
    assert _mlp(lib, eps=0.0) == INVALID
    assert _mlp(lib, eps=float("nan")) == INVALID
    assert _mlp(lib, act=7) == INVALID
    assert _mlp(lib, dtype=0, out=1) == INVALID        # f32 storage cannot write bf16
    assert _mlp(lib, dtype=5) == INVALID
    assert _mlp(lib, F=1000, t=3) == UNSUPPORTED      # F % t
    assert _mlp(lib, F=1020, t=2) == UNSUPPORTED      # shard width % 8
    assert _mlp(lib, H=260) == UNSUPPORTED            # H % 8
    assert _mlp(lib, H=16392) == UNSUPPORTED          # above the LayerNorm row limit
    assert _mlp(lib, ws_bytes=100) == WS_SMALL
    pa, ka = _ptrs(2)
    ka[1] = None
    assert _mlp(lib, A=(pa, ka)) == INVALID            # null shard


def test_attention_argument_checks(lib):
    pq, kq = _ptrs(4)
    po, ko = _ptrs(4)

    def call(S=2048, H=8192, nh=64, d=128, t=4, dtype=1, ws_bytes=1 << 34):
        return lib.tp_qkv_attn_oproj_forward(S, H, nh, d, t, dtype, 1, ctypes.c_void_p(FAKE), pq, po, None, None,
                                             1e-5, ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ws_bytes, None)
    assert call(dtype=0) == INVALID
    assert call(d=64, H=4096) == UNSUPPORTED
    assert call(nh=63, H=63 * 128) == UNSUPPORTED      # nh % t
    assert call(H=8000) == UNSUPPORTED                 # H != nh * d
    assert call(S=2000) == UNSUPPORTED                 # S % 128
    assert call(ws_bytes=10) == WS_SMALL


def test_linear_and_layernorm_argument_checks(lib):
    pw, kw = _ptrs(2)
    assert lib.tp_linear_column_forward(64, 100, 256, 2, 1, 0, ctypes.c_void_p(FAKE), pw, 0,
                                        ctypes.c_void_p(FAKE), None) == UNSUPPORTED
    assert lib.tp_linear_column_forward(64, 128, 250, 2, 1, 0, ctypes.c_void_p(FAKE), pw, 0,
                                        ctypes.c_void_p(FAKE), None) == UNSUPPORTED
    assert lib.tp_linear_row_forward(64, 100, 256, 2, 1, 0, ctypes.c_void_p(FAKE), pw, ctypes.c_void_p(FAKE),
                                     None, 0, None) == UNSUPPORTED
    assert lib.tp_linear_row_forward(64, 128, 256, 0, 1, 0, ctypes.c_void_p(FAKE), pw, ctypes.c_void_p(FAKE),
                                     None, 0, None) == INVALID
    assert lib.tp_reduce_residual_layernorm(8, 12, 0, None, ctypes.c_void_p(FAKE), 1, None, None, 1e-5,
                                            ctypes.c_void_p(FAKE), 1, None) == UNSUPPORTED
    assert lib.tp_reduce_residual_layernorm(8, 16, 1, None, ctypes.c_void_p(FAKE), 1, None, None, 1e-5,
                                            ctypes.c_void_p(FAKE), 1, None) == INVALID


def test_training_argument_checks(lib):
    S, H, F, t = 128, 256, 1024, 2
    pa, ka = _ptrs(t)
    pb, kb = _ptrs(t)
    pda, kda = _ptrs(t)
    pdb, kdb = _ptrs(t)
    st_bytes = lib.tp_mlp_train_state_bytes(S, H, F, t, 1)
    assert st_bytes == 2 * S * F * 2 + S * H * 4 + S * 8  # U, G, V and the LayerNorm's row statistics
    assert lib.tp_mlp_train_state_bytes(S, H, F, t, 0) == 0      # f32 storage has no training path
    ws_bytes = lib.tp_mlp_backward_workspace_bytes(S, H, F, t, 1)
    assert ws_bytes >= S * H * 2 + S * F * 2 + S * H * 4
    P = ctypes.c_void_p(FAKE)

    def fwd(dtype=1, state_bytes=st_bytes, act=1):
        return lib.tp_mlp_forward_train(S, H, F, t, dtype, 1, P, pa, pb, None, None, 1e-5, act, P, P, state_bytes,
                                        None)

    def bwd(dtype=1, dY=P, state_bytes=st_bytes, ws=ws_bytes, dA=pda):
        return lib.tp_mlp_backward(S, H, F, t, dtype, P, pa, pb, None, 1e-5, 1, P, state_bytes, dY, P, dA, pdb,
                                   None, None, P, ws, None)

    assert fwd(dtype=0) == UNSUPPORTED
    assert fwd(act=9) == INVALID
    assert fwd(state_bytes=st_bytes - 1) == WS_SMALL
    assert bwd(dtype=0) == UNSUPPORTED
    assert bwd(dY=None) == INVALID
    assert bwd(dY=ctypes.c_void_p(FAKE + 8)) == INVALID             # misaligned
    assert bwd(dA=None) == INVALID
    assert bwd(state_bytes=1) == WS_SMALL
    assert bwd(ws=ws_bytes - 1) == WS_SMALL


def test_gemm_tile_override_checks(lib):
    try:
        for bad in (-32, 64, 100, 160, 224, 300, 544):
            assert lib.tp_set_gemm_tile_n(bad) == INVALID
        for good in (128, 256, 288, 480, 512, 0):
            assert lib.tp_set_gemm_tile_n(good) == OK
    finally:
        lib.tp_set_gemm_tile_n(0)


def test_weight_layout_argument_checks(lib):
    pw, kw = _ptrs(2)
    X, Y = ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE)
    for layout in (-1, 2):
        assert lib.tp_linear_column_forward_ex(64, 128, 256, 2, 1, 0, layout, X, pw, 0, Y, None) == INVALID
        assert lib.tp_linear_row_forward_ex(64, 128, 256, 2, 1, 0, layout, X, pw, Y, None, 0, None) == INVALID
        assert lib.tp_mlp_forward_ex(64, 128, 256, 2, 1, 1, layout, X, pw, pw, None, None, 1e-5, 1, Y, X,
                                     1 << 30, None) == INVALID
        assert lib.tp_qkv_attn_oproj_forward_ex(128, 256, 2, 128, 2, 1, 1, layout, X, pw, pw, None, None, 1e-5,
                                                Y, X, 1 << 30, None) == INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="only meaningful without a CUDA device")
def test_valid_call_without_device_reports_no_device(lib):
    assert _mlp(lib) == NO_DEVICE


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        L.lib()
