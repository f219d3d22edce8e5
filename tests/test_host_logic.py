"""Host-side logic pinned to numbers the pages print and to closed forms:
shard shapes, payload bytes, heads per shard, workload FLOP counts, the row
sample and the seeded generator's determinism."""
from __future__ import annotations

import json
import os

import pytest
import torch

from megatron_tensor_transformer_gelu_b200 import synth
from megatron_tensor_transformer_gelu_b200.workloads import HEADLINE, WORKLOADS

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "pages_printed_numbers.json")


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_column_split_example_shapes(golden):
    g = golden["column_split_example"]
    W = torch.empty(*g["W_shape"], device="meta")
    shards = synth.split_columns(W, g["shards"])
    assert [list(s.shape) for s in shards] == [g["shard_shape"]] * g["shards"]


def test_reduction_payload_bytes(golden):
    g = golden["allreduce_payload_tp2"]
    payload = g["S"] * g["H"] * g["bytes_per_element"] * g["ring_factor"]
    assert payload / 1e6 == pytest.approx(g["printed_MB"], abs=0.05)
    assert 2 * payload / 1e6 == pytest.approx(g["printed_block_MB"], abs=0.5)
    # the headline workload's [S, H] bf16 activation is the same shape
    w = WORKLOADS[HEADLINE]
    assert (w.S, w.H) == (g["S"], g["H"])


def test_heads_per_shard(golden):
    g = golden["heads_per_shard_example"]
    w = WORKLOADS["attn_s2048_h8192_64x128"]
    assert (w.nh, w.t) == (g["heads"], g["tp"])
    H = w.nh * w.d
    Wqkv = torch.empty(H, 3 * H, device="meta")
    shards = synth.split_qkv_by_head(Wqkv, w.nh, w.d, w.t)
    assert all(s.shape[1] == 3 * g["heads_per_shard"] * w.d for s in shards)


def test_qkv_shard_columns_follow_heads():
    nh, d, t = 4, 2, 2
    H = nh * d
    Wqkv = torch.arange(3 * H, dtype=torch.float32).repeat(3, 1)  # column index as value
    s1 = synth.split_qkv_by_head(Wqkv, nh, d, t)[1]
    # shard 1 holds heads 2..3 of Q (cols 4..7), of K (12..15), of V (20..23)
    assert s1[0].tolist() == [4, 5, 6, 7, 12, 13, 14, 15, 20, 21, 22, 23]


def test_workload_flops():
    assert WORKLOADS["mlp_s2048_h4096_f16384"].flops == 549_755_813_888        # 549.8 GFLOP
    assert WORKLOADS["mlp_s4096_h12288_f49152"].flops == 2 * 2 * 4096 * 12288 * 49152
    assert WORKLOADS["linear_col_4096x4096x8192"].flops == 2 * 4096 * 4096 * 8192
    a = WORKLOADS["attn_s2048_h8192_64x128"]
    assert a.flops == 2 * 2048 * 8192 * 3 * 8192 + 4 * 2048 * 2048 * 128 * 64 + 2 * 2048 * 8192 * 8192


def test_training_workload_flops():
    """A training step counts every product of the forward and the backward:
    the MLP's 2 forward GEMMs plus dU, dX, dA, dB (each 2 S H F); the attention
    sublayer's forward plus dO, dWo, the five per-head products of the softmax
    attention's backward (each 2 S^2 d per head) and dX, dWqkv."""
    S, H, F = 2048, 4096, 16384
    assert WORKLOADS["mlp_train_s2048_h4096_f16384"].flops == 6 * 2 * S * H * F
    S, H, nh, d = 2048, 8192, 64, 128
    qkv, oproj = 2 * S * H * 3 * H, 2 * S * H * H
    fwd = qkv + 4 * S * S * d * nh + oproj
    bwd = 2 * oproj + 5 * 2 * S * S * d * nh + 2 * qkv
    assert WORKLOADS["attn_train_s2048_h8192_64x128"].flops == fwd + bwd
    assert round((fwd + bwd) / 1e9, 1) == 3779.6


def test_row_sample_deterministic_and_bounded():
    r1 = synth.row_sample(2048, 1)
    r2 = synth.row_sample(2048, 1)
    assert r1 == r2 and len(r1) == 64 and r1[0] == 0 and r1[-1] == 2047
    assert r1 == sorted(set(r1))
    assert synth.row_sample(10, 1) == list(range(10))


def test_generator_is_seeded_and_scaled():
    a = synth.gen_mlp(64, 128, 256, seed=3, dtype=torch.float32)
    b = synth.gen_mlp(64, 128, 256, seed=3, dtype=torch.float32)
    assert torch.equal(a.A, b.A) and torch.equal(a.X, b.X)
    # N(0, 1/fan_in): A has fan_in H = 128, B has fan_in F = 256
    assert a.A.std().item() == pytest.approx(128 ** -0.5, rel=0.05)
    assert a.B.std().item() == pytest.approx(256 ** -0.5, rel=0.05)
    c = synth.gen_mlp(64, 128, 256, seed=4, dtype=torch.float32)
    assert not torch.equal(a.A, c.A)


def test_bf16_storage_is_rounded_fp32_draw():
    f = synth.gen_mlp(8, 16, 32, seed=5, dtype=torch.float32)
    h = synth.gen_mlp(8, 16, 32, seed=5, dtype=torch.bfloat16)
    assert torch.equal(f.X.to(torch.bfloat16), h.X)
    assert torch.equal(f.A.to(torch.bfloat16), h.A)


def test_bench_kernel_table_roofline_arithmetic():
    """bench.py's per-kernel roofline: algorithmic work per launch (work per
    step / launches per step) over the mean event-timed launch duration; the
    f32 CUDA-core kind against SMs x 128 FMA x 2 x clock."""
    import bench
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0, "source": "measured"}
    steps = 4
    # 2 GEMM launches per step of 1e12 FLOP each, 2 ms each; 1 LayerNorm launch of 6.5e9 B taking 1 ms
    prof = {"gemm_tcgen05": (8, 8, 16.0), "reduce_residual_layernorm": (4, 4, 4.0), "attention_fwd": (0, 0, 0.0)}
    work = {"gemm_tcgen05": 2e12, "reduce_residual_layernorm": 6.5e9}
    k = bench.kernel_table(prof, work, steps, peaks)
    assert k["gemm_tcgen05"]["achieved"] == pytest.approx(500.0)
    assert k["gemm_tcgen05"]["frac"] == pytest.approx(500.0 / 1600.0, abs=1e-4)
    assert k["gemm_tcgen05"]["flops_per_launch"] == 1e12
    assert k["reduce_residual_layernorm"]["achieved"] == pytest.approx(6500.0)
    assert k["reduce_residual_layernorm"]["frac"] == pytest.approx(1.0)
    assert k["gemm_tcgen05"]["share_of_step"] == pytest.approx(0.8)
    dom, roof = bench.dominant(k, peaks, "none")
    assert dom == "gemm_tcgen05" and roof["frac_of_sustained"] == pytest.approx(500.0 / 1400.0, abs=1e-4)
    # f32 FMA peak of 148 SMs at 1965 MHz: 148 * 128 * 2 * 1.965e9 = 74.45 TFLOP/s
    assert bench.alu_peak(148, 1965.0) == pytest.approx(74.449, abs=1e-3)
    ka = bench.kernel_table({"gemm_simt_f32": (2, 2, 0.004)}, {"gemm_simt_f32": 1.34e8}, 1, peaks, 74.449)
    assert ka["gemm_simt_f32"]["bound"] == "alu"
    assert ka["gemm_simt_f32"]["achieved"] == pytest.approx(1.34e8 / 2 / 2e-6 / 1e12, abs=0.01)
