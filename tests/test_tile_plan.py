"""Host logic of the GEMM tile plan (tp_gemm_plan: the choice the next launch
of a shape gets), pinned on the GEMM shapes of the workloads.  No device is
touched.  The expected picks follow from the cost model the header documents:
waves x k-blocks x time per k-block (relative time per MAC 1.0 at 256 columns
down to 0.75 at 512), plus the epilogue each wave but the last exposes for
wide tiles (doubled for epilogues that store or read a second operand), plus
the f32 slot traffic of a K split; a wide tile must buy 2 %."""
from __future__ import annotations

import pytest

from megatron_tensor_transformer_gelu_b200 import _lib as L
from megatron_tensor_transformer_gelu_b200 import build as B

PAIRS = 74  # co-resident CTA pairs on a 148-SM B200


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()
    L.lib()
    L.set_gemm_tile_n(0)


# (name, M, t, row_mode, shard_k, shard_n, out_f32, b_kmajor, heavy_epilogue, max_splits) -> (tile_n, splits)
CASES = [
    # MLP S2048 H4096 F16384 t4: 256 tiles of 512 columns in 3.46 waves beat 512 tiles of 256 in 7
    ("mlp GEMM1", 2048, 4, 0, 4096, 4096, 0, 0, 0, 1, (512, 1)),
    # row split over 4 shards: 64 tiles of 512 columns, one wave, no K split
    ("mlp GEMM2", 2048, 4, 1, 4096, 4096, 1, 0, 0, 4, (512, 1)),
    # attention S2048 H8192 t4: QKV (3 x 2048 columns per shard) and O projection
    ("QKV", 2048, 4, 0, 8192, 6144, 0, 0, 0, 1, (512, 1)),
    ("O projection", 2048, 4, 1, 2048, 8192, 1, 0, 0, 4, (512, 1)),
    # large MLP S4096 H12288 F49152 t8
    ("large GEMM1", 4096, 8, 0, 12288, 6144, 0, 0, 0, 1, (512, 1)),
    ("large GEMM2", 4096, 8, 1, 6144, 12288, 1, 0, 0, 4, (512, 1)),
    # training forward GEMM1 also stores U: its exposed epilogue doubles, 256 stays
    ("train GEMM1 + U store", 2048, 4, 0, 4096, 4096, 0, 0, 1, 1, (256, 1)),
    # dU = (dZ B^T) * Act'(U): K-major B, reads U in the epilogue
    ("train dU", 2048, 4, 0, 4096, 4096, 0, 1, 1, 1, (256, 1)),
    # attention backward: dV/dQ/dK of a group of 8 heads (N = d = 128, N-major B): narrow tiles
    ("attn dV (8 heads)", 2048, 8, 0, 2048, 128, 0, 0, 0, 1, (128, 1)),
    # the score GEMM of a group (K = 128, K-major B, softmax epilogue): 256
    ("attn P (8 heads)", 2048, 8, 0, 128, 2048, 0, 1, 1, 1, (256, 1)),
    # a K-major B never gets narrow tiles (its box is 128 rows per CTA)
    ("K-major 128 columns", 2048, 1, 0, 2048, 128, 0, 1, 0, 1, (256, 1)),
    # single CTAs (M < 129): 256 unless narrow
    ("single-CTA", 100, 2, 0, 512, 1024, 0, 0, 0, 1, (256, 1)),
    ("single-CTA narrow", 100, 2, 0, 512, 64, 0, 0, 0, 1, (128, 1)),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_plan_of_workload_gemms(case):
    _, M, t, row, sk, sn, f32, bk, heavy, ms, want = case
    assert L.gemm_plan(M, t, row, sk, sn, f32, bk, heavy, PAIRS, ms) == want


def test_k_split_fills_idle_pairs():
    """A row-split GEMM with few tiles and a long K loop (f32 out): splitting K
    puts the idle pairs to work; never with bf16 output or max_splits = 1."""
    tn, sp = L.gemm_plan(512, 4, 1, 4096, 1024, 1, 0, 0, PAIRS, 4)
    assert sp > 1 and tn == 256
    assert L.gemm_plan(512, 4, 1, 4096, 1024, 0, 0, 0, PAIRS, 4)[1] == 1
    assert L.gemm_plan(512, 4, 1, 4096, 1024, 1, 0, 0, PAIRS, 1)[1] == 1


def test_override_is_what_the_next_launch_gets():
    try:
        L.set_gemm_tile_n(480)
        assert L.gemm_plan(2048, 4, 1, 4096, 4096, 1, 0, 0, PAIRS, 4) == (480, 1)  # f32: 32-column steps
        assert L.gemm_plan(2048, 4, 0, 4096, 4096, 0, 0, 0, PAIRS, 1) == (512, 1)  # bf16: rounded up to 64
        assert L.gemm_plan(100, 2, 0, 512, 1024, 0, 0, 0, PAIRS, 1) == (256, 1)    # single CTAs: no wide tiles
        L.set_gemm_tile_n(128)
        assert L.gemm_plan(2048, 4, 0, 4096, 4096, 0, 0, 0, PAIRS, 1) == (128, 1)
        assert L.gemm_plan(100, 2, 0, 512, 1024, 0, 0, 0, PAIRS, 1) == (128, 1)
    finally:
        L.set_gemm_tile_n(0)
    assert L.gemm_plan(2048, 4, 0, 4096, 4096, 0, 0, 0, PAIRS, 1) == (512, 1)


def test_bad_arguments():
    import ctypes
    tn, sp = ctypes.c_int(), ctypes.c_int()
    lib = L.lib()
    for args in [(0, 4, 0, 64, 64), (64, 0, 0, 64, 64), (64, 9, 0, 64, 64), (64, 4, 0, 0, 64), (64, 4, 0, 64, 0)]:
        assert lib.tp_gemm_plan(*args, 0, 0, 0, PAIRS, 1, ctypes.byref(tn), ctypes.byref(sp)) == 1
    assert lib.tp_gemm_plan(64, 4, 0, 64, 64, 0, 0, 0, 0, 1, ctypes.byref(tn), ctypes.byref(sp)) == 1
    assert lib.tp_gemm_plan(64, 4, 0, 64, 64, 0, 0, 0, PAIRS, 1, None, ctypes.byref(sp)) == 1


# With the sublayers' spare partial-sum slots (3 x S x H x 4 bytes) as stream-K
# scratch: (tile_n, splits, stream_k, pairs).  Stream-K (whole waves, then the
# remainder tiles split along K) wins where the last wave leaves pairs idle:
# 64 or 128 tiles of 512 columns on 74 pairs, 256 or 384 in 3.46 / 5.19 waves.
# The large MLP's first GEMM (1536 tiles, 20.75 waves) gains under 2 % and
# keeps whole tiles.
SK_CASES = [
    ("mlp GEMM1", 2048, 4, 0, 4096, 4096, 0, 1, 2048 * 4096, (512, 1, 1, 74)),
    ("mlp GEMM2", 2048, 4, 1, 4096, 4096, 1, 4, 2048 * 4096, (512, 1, 1, 74)),
    ("QKV", 2048, 4, 0, 8192, 6144, 0, 1, 2048 * 8192, (512, 1, 1, 74)),
    ("O projection", 2048, 4, 1, 2048, 8192, 1, 4, 2048 * 8192, (512, 1, 1, 74)),
    ("large GEMM1", 4096, 8, 0, 12288, 6144, 0, 1, 4096 * 12288, (512, 1, 0, 0)),
    ("large GEMM2", 4096, 8, 1, 6144, 12288, 1, 4, 4096 * 12288, (512, 1, 1, 74)),
    # too little scratch for 74 partial blocks of 256 x 256: the K split stays
    ("small row split", 1024, 4, 1, 1024, 1024, 1, 4, 1024 * 1024, (256, 4, 0, 0)),
]


@pytest.mark.parametrize("case", SK_CASES, ids=[c[0] for c in SK_CASES])
def test_stream_k_plan_of_workload_gemms(case):
    _, M, t, row, sk, sn, f32, ms, sh, want = case
    try:
        L.set_gemm_stream_k(2)  # the cost model (stream-K is off by default)
        assert L.gemm_plan_sk(M, t, row, sk, sn, f32, max_splits=ms, sk_area_bytes=3 * sh * 4) == want
    finally:
        L.set_gemm_stream_k(0)


def test_stream_k_switch():
    try:
        # the default: whole tiles even with scratch
        L.set_gemm_stream_k(0)
        assert L.gemm_plan_sk(2048, 4, 1, 4096, 4096, 1, max_splits=4, sk_area_bytes=3 * 2048 * 4096 * 4)[2] == 0
        # forced: as many pairs as the scratch holds 256 x 256 f32 blocks for (+ one flag each)
        L.set_gemm_stream_k(1)
        area = 10 * 2 * 128 * 256 * 4 + 256 + 10 * 2 * 8
        # 3 x 8 = 24 tiles on 10 pairs: 2 whole waves, 4 remainder tiles split
        tn, sp, on, pairs = L.gemm_plan_sk(600, 2, 0, 520, 1000, 0, sk_area_bytes=area)
        assert (tn, sp, on, pairs) == (256, 1, 1, 10)
        # 3 x 10 = 30 tiles on 10 pairs: whole waves only, nothing to split
        assert L.gemm_plan_sk(600, 2, 0, 520, 1120, 0, sk_area_bytes=area)[2] == 0
        # no scratch, no stream-K
        assert L.gemm_plan_sk(600, 2, 0, 520, 1000, 0, sk_area_bytes=0)[2] == 0
        with pytest.raises(L.TPError):
            L.set_gemm_stream_k(3)
    finally:
        L.set_gemm_stream_k(0)


# ---------------------------------------------- attention key-split plan
def _split_bytes(R):
    r256 = lambda x: (x + 255) // 256 * 256
    return r256(R * 8 * 32 * 128 * 4) + r256(R * 8 * 64 * 4) + R * 8 * 2 * 8


def test_attn_split_plan_of_the_workload():
    # 64 heads x 8 query blocks = 512 units on 148 SMs: 3 waves + 68 units,
    # which run as 136 half-key CTAs (8 + 8 key blocks)
    assert L.attn_split_plan(2048, 64, slots=148, mode=1) == (444, 68, 8)
    assert L.attn_split_plan(2048, 64, slots=148, mode=0) == (512, 0, 0)
    assert L.attn_split_plan(2048, 64, slots=148, mode=2) == (0, 512, 8)
    # exactly enough scratch, and one byte short
    assert L.attn_split_plan(2048, 64, 148, 1, _split_bytes(68)) == (444, 68, 8)
    assert L.attn_split_plan(2048, 64, 148, 1, _split_bytes(68) - 1) == (512, 0, 0)


def test_attn_split_plan_edges():
    # the remainder does not fit twice in a wave (248 = 148 + 100): no split
    assert L.attn_split_plan(2048, 31, slots=148, mode=1) == (248, 0, 0)
    # whole waves only: nothing to split
    assert L.attn_split_plan(2048, 37, slots=148, mode=1) == (296, 0, 0)
    # fewer units than SMs: every unit is in the partial wave
    assert L.attn_split_plan(1024, 16, slots=148, mode=1) == (0, 64, 4)
    # fewer than 4 key blocks: not worth it by default, possible when forced
    assert L.attn_split_plan(384, 2, slots=148, mode=1) == (4, 0, 0)
    assert L.attn_split_plan(384, 2, slots=148, mode=2) == (0, 4, 1)
    # one key block cannot be halved
    assert L.attn_split_plan(128, 2, slots=148, mode=2) == (2, 0, 0)
    assert L.attn_split_plan(0, 2, slots=148, mode=2) == (0, 0, 0)
    for args in ((-1, 2, 148, 1), (256, 0, 148, 1), (256, 2, 0, 1), (256, 2, 148, 3)):
        with pytest.raises(L.TPError):
            L.attn_split_plan(*args)
    with pytest.raises(L.TPError):
        L.set_attn_kv_split(3)


# --------------------------------------- weight-gradient GEMMs (M-major A)
# (M, t, shard_k, shard_n): the MLP's dA = X^T dU and dB = G^T dZ, the attention
# backward's dWo = O^T dZ and dWqkv = X^T dQKV, all f32 out.  With an M-major
# A the 256-column tiles cost 10 % more per k-block (measured), so the wide
# tiles win; the same shapes with a K-major A keep 256.
WGRAD_CASES = [("mlp dA", 4096, 4, 2048, 4096), ("mlp dB", 16384, 1, 2048, 4096),
               ("attn dWo", 8192, 1, 2048, 8192), ("attn dWqkv", 8192, 4, 2048, 6144)]


@pytest.mark.parametrize("case", WGRAD_CASES, ids=[c[0] for c in WGRAD_CASES])
def test_weight_gradient_gemms_take_wide_tiles(case):
    _, M, t, sk, sn = case
    assert L.gemm_plan_ex(M, t, 0, sk, sn, True, a_mnmajor=True) == (512, 1, 0, 0)
    assert L.gemm_plan_ex(M, t, 0, sk, sn, True, a_mnmajor=False) == (256, 1, 0, 0)
    assert L.gemm_plan_sk(M, t, 0, sk, sn, True) == L.gemm_plan_ex(M, t, 0, sk, sn, True)
