"""The workloads the sublayer is checked and measured on (sizes, shard counts,
storage types, seeds).  FLOP counts take 2 per multiply-accumulate of the GEMMs
and the attention matmuls only; activation, softmax and LayerNorm work is
elementwise and left out of the count."""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "mlp" | "mlp_train" | "attn" | "attn_train" | "linear_col" | "linear_row"
    dtype: str           # "f32" | "bf16"  (storage of X and weights)
    t: int               # shard count
    seed: int = 0
    S: int = 0
    H: int = 0
    F: int = 0
    nh: int = 0
    d: int = 0
    M: int = 0
    K: int = 0
    N: int = 0
    act: str = "gelu_tanh"
    t_sweep: tuple = field(default_factory=tuple)

    @property
    def flops(self) -> int:
        if self.kind == "mlp":
            return 2 * 2 * self.S * self.H * self.F
        if self.kind == "mlp_train":
            # forward (X A, G B) + backward (dZ B^T, dU A^T, X^T dU, G^T dZ)
            return 6 * 2 * self.S * self.H * self.F
        if self.kind in ("attn", "attn_train"):
            S, H = self.S, self.H
            qkv = 2 * S * H * 3 * H
            att = 2 * 2 * S * S * self.d * self.nh
            oproj = 2 * S * H * H
            if self.kind == "attn":
                return qkv + att + oproj
            # + backward: dO and dWo (2 x oproj), per head the rebuilt scores,
            # dV, dP, dQ and dK (5 x att / 2), dX and dWqkv (2 x qkv)
            return qkv + att + oproj + 2 * oproj + 5 * att // 2 + 2 * qkv
        return 2 * self.M * self.K * self.N


WORKLOADS = {
    w.name: w
    for w in [
        Workload("mlp_tiny_f32", "mlp", "f32", t=2, seed=0, S=128, H=256, F=1024,
                 t_sweep=(1, 2, 4)),
        Workload("linear_col_4096x4096x8192", "linear_col", "bf16", t=2, seed=0,
                 M=4096, K=4096, N=8192, act="none", t_sweep=(1, 2, 4)),
        Workload("linear_row_4096x4096x8192", "linear_row", "bf16", t=2, seed=0,
                 M=4096, K=4096, N=8192, act="none", t_sweep=(1, 2, 4)),
        Workload("mlp_s2048_h4096_f16384", "mlp", "bf16", t=4, seed=0,
                 S=2048, H=4096, F=16384, t_sweep=(1, 2, 4, 8)),
        Workload("attn_s2048_h8192_64x128", "attn", "bf16", t=4, seed=0,
                 S=2048, H=8192, nh=64, d=128, act="none", t_sweep=(1, 2, 4, 8)),
        Workload("mlp_s4096_h12288_f49152", "mlp", "bf16", t=8, seed=7,
                 S=4096, H=12288, F=49152, t_sweep=(8,)),
        # One training step of the headline sublayer: forward keeping U/G/V,
        # then the backward pass (all gradients).
        Workload("mlp_train_s2048_h4096_f16384", "mlp_train", "bf16", t=4, seed=0,
                 S=2048, H=4096, F=16384, t_sweep=(4,)),
        # One training step of the attention sublayer: forward keeping state,
        # then the backward pass.
        Workload("attn_train_s2048_h8192_64x128", "attn_train", "bf16", t=4, seed=0,
                 S=2048, H=8192, nh=64, d=128, act="none", t_sweep=(4,)),
    ]
}

# The workload the headline throughput is quoted on.
HEADLINE = "mlp_s2048_h4096_f16384"
