// fp32 path on the CUDA cores, for fp32 storage.  tf32 tensor-core products
// would miss the fp32 tolerance, so the fp32 sublayer runs as FFMA tiles.
//
// Same sharding semantics as the tensor-core GEMM: column mode writes shard s
// into its column slice of C (concatenation as a layout, "按列切分"); row mode
// walks the shards along K and sums their partial products in registers
// ("按行切分" / "外积和切分").
#pragma once
#include <cuda_runtime.h>

#include "gemm_tcgen05.cuh"

namespace tp {

struct SimtArgs {
  const float* A;                 // [M, K_total], row stride lda
  long long lda;
  const float* B[MAX_SHARDS];     // shard s: [shard_k, shard_n] row-major
  float* C;                       // [M, ...], row stride ldc
  long long ldc;
  int M, N, K;                    // N: total output columns, K: total reduction length
  int row_mode;
  int shard_n, shard_k;
  int act;
  int b_kmajor;                   // shards stored [shard_n, shard_k] (nn.Linear [out, in])
};

namespace simt {
constexpr int TM = 64, TN = 64, TK = 16, THREADS = 256;
}

__device__ __forceinline__ float apply_act_precise(float u, int act) {
  if (act == ACT_GELU_TANH) {
    const float k0 = 0.7978845608028654f;
    return 0.5f * u * (1.0f + tanhf(k0 * (u + 0.044715f * u * u * u)));
  } else if (act == ACT_GELU_ERF) {
    return 0.5f * u * (1.0f + erff(u * 0.7071067811865476f));
  } else if (act == ACT_RELU) {
    return fmaxf(u, 0.0f);
  }
  return u;
}

__device__ __forceinline__ float simt_b(const SimtArgs& p, int k, int n) {
  int s, kk, nn;
  if (p.row_mode) {
    s = k / p.shard_k;
    kk = k - s * p.shard_k;
    nn = n;
  } else {
    s = n / p.shard_n;
    kk = k;
    nn = n - s * p.shard_n;
  }
  return p.b_kmajor ? p.B[s][static_cast<long long>(nn) * p.shard_k + kk]
                    : p.B[s][static_cast<long long>(kk) * p.shard_n + nn];
}

// 64x64 output tile per block, 4x4 per thread, K in steps of 16 through smem.
__global__ void __launch_bounds__(simt::THREADS) simt_gemm_f32_kernel(const SimtArgs p) {
  using namespace simt;
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int m0 = blockIdx.y * TM;
  const int n0 = blockIdx.x * TN;
  const int tx = threadIdx.x % 16;   // column group
  const int ty = threadIdx.x / 16;   // row group
  float acc[4][4] = {};
  for (int k0 = 0; k0 < p.K; k0 += TK) {
    for (int i = threadIdx.x; i < TM * TK; i += THREADS) {
      const int r = i / TK, kk = i % TK;
      const int gm = m0 + r, gk = k0 + kk;
      As[kk][r] = (gm < p.M && gk < p.K) ? p.A[static_cast<long long>(gm) * p.lda + gk] : 0.0f;
    }
    for (int i = threadIdx.x; i < TK * TN; i += THREADS) {
      const int kk = i / TN, c = i % TN;
      const int gk = k0 + kk, gn = n0 + c;
      Bs[kk][c] = (gk < p.K && gn < p.N) ? simt_b(p, gk, gn) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn < p.N) p.C[static_cast<long long>(gm) * p.ldc + gn] = apply_act_precise(acc[i][j], p.act);
    }
  }
}

}  // namespace tp
