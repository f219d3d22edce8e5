// fp32 path on the CUDA cores, for fp32 storage.  tf32 tensor-core products
// would miss the fp32 tolerance, so the fp32 sublayer runs as FFMA tiles.
//
// Same sharding semantics as the tensor-core GEMM: column mode writes shard s
// into its column slice of C (concatenation as a layout, "按列切分"); row mode
// walks the shards along K and sums their partial products in registers
// ("按行切分" / "外积和切分").
//
// The f32 workloads are small (the tiny MLP is 0.13 GFLOP), so the kernel is
// shaped for latency: 32 x 32 output tiles (many CTAs), 128-bit loads, the
// next K chunk's loads issued before the current chunk's FMAs, and (row mode,
// no activation) an optional split of the K range over blockIdx.z, each split
// writing its own f32 slot that the reduce + LayerNorm kernel adds in order.
#pragma once
#include <cuda_runtime.h>

#include "gemm_tcgen05.cuh"

namespace tp {

struct SimtArgs {
  const float* A;                 // [M, K_total], row stride lda
  long long lda;
  const float* B[MAX_SHARDS];     // shard s: [shard_k, shard_n] row-major
  float* C;                       // [M, ...], row stride ldc; split z at C + z * slot_stride
  long long ldc;
  long long slot_stride;
  int M, N, K;                    // N: total output columns, K: total reduction length
  int row_mode;
  int shard_n, shard_k;
  int act;
  int b_kmajor;                   // shards stored [shard_n, shard_k] (nn.Linear [out, in])
  int splits;                     // K range split over blockIdx.z (act must be none when > 1)
};

namespace simt {
constexpr int TM = 32, TN = 32, TK = 32, THREADS = 128;
constexpr int PAD = 4;  // smem row padding (floats): keeps the transposed stores off one bank
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

// Four consecutive B values along n (N-major storage) at reduction index k and
// output column n (n % 4 == 0), or along k (K-major storage, k % 4 == 0).
// Shard widths are multiples of 8, so the four never straddle two shards.
__device__ __forceinline__ const float* simt_b_ptr(const SimtArgs& p, int k, int n) {
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
  return p.b_kmajor ? p.B[s] + static_cast<long long>(nn) * p.shard_k + kk
                    : p.B[s] + static_cast<long long>(kk) * p.shard_n + nn;
}

// 32 x 32 output tile per CTA of 128 threads, 2 x 4 outputs per thread, K in
// chunks of 32 staged through shared memory.  Every K and N here is a
// multiple of 8 (the entry points check it), so a 128-bit load is either
// wholly inside the matrix or wholly outside.
__global__ void __launch_bounds__(simt::THREADS) simt_gemm_f32_kernel(const SimtArgs p) {
  using namespace simt;
  __shared__ __align__(16) float As[TK][TM + PAD];
  __shared__ __align__(16) float Bs[TK][TN + PAD];
  const int m0 = blockIdx.y * TM;
  const int n0 = blockIdx.x * TN;
  const int tid = threadIdx.x;
  const int ty = tid / 8;   // rows 2 ty, 2 ty + 1
  const int tx = tid % 8;   // columns 4 tx .. 4 tx + 3
  const int nch = (p.K + TK - 1) / TK;
  const int c0 = static_cast<int>(static_cast<long long>(blockIdx.z) * nch / p.splits);
  const int c1 = static_cast<int>(static_cast<long long>(blockIdx.z + 1) * nch / p.splits);

  // Each thread moves 2 float4 of A and 2 of B per chunk.
  float4 ra[2], rb[2];
  auto load_chunk = [&](int c) {
    const int k0 = c * TK;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int i = tid + j * THREADS;        // 0..255
      {  // A: row i / 8, k quad i % 8
        const int gm = m0 + i / 8, gk = k0 + (i % 8) * 4;
        ra[j] = (gm < p.M && gk < p.K) ? *reinterpret_cast<const float4*>(p.A + static_cast<long long>(gm) * p.lda + gk)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (!p.b_kmajor) {  // B: k row i / 8, n quad i % 8
        const int gk = k0 + i / 8, gn = n0 + (i % 8) * 4;
        rb[j] = (gk < p.K && gn < p.N) ? *reinterpret_cast<const float4*>(simt_b_ptr(p, gk, gn))
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
      } else {            // B K-major: n row i / 8, k quad i % 8
        const int gn = n0 + i / 8, gk = k0 + (i % 8) * 4;
        rb[j] = (gk < p.K && gn < p.N) ? *reinterpret_cast<const float4*>(simt_b_ptr(p, gk, gn))
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  auto store_chunk = [&]() {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int i = tid + j * THREADS;
      const int r = i / 8, q = (i % 8) * 4;
      As[q + 0][r] = ra[j].x;
      As[q + 1][r] = ra[j].y;
      As[q + 2][r] = ra[j].z;
      As[q + 3][r] = ra[j].w;
      if (!p.b_kmajor) {
        *reinterpret_cast<float4*>(&Bs[r][q]) = rb[j];
      } else {
        Bs[q + 0][r] = rb[j].x;
        Bs[q + 1][r] = rb[j].y;
        Bs[q + 2][r] = rb[j].z;
        Bs[q + 3][r] = rb[j].w;
      }
    }
  };

  float acc[2][4] = {};
  if (c0 < c1) load_chunk(c0);
  for (int c = c0; c < c1; ++c) {
    store_chunk();
    __syncthreads();
    if (c + 1 < c1) load_chunk(c + 1);  // in flight while this chunk's FMAs run
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      const float2 a = *reinterpret_cast<const float2*>(&As[kk][ty * 2]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      acc[0][0] = fmaf(a.x, b.x, acc[0][0]);
      acc[0][1] = fmaf(a.x, b.y, acc[0][1]);
      acc[0][2] = fmaf(a.x, b.z, acc[0][2]);
      acc[0][3] = fmaf(a.x, b.w, acc[0][3]);
      acc[1][0] = fmaf(a.y, b.x, acc[1][0]);
      acc[1][1] = fmaf(a.y, b.y, acc[1][1]);
      acc[1][2] = fmaf(a.y, b.z, acc[1][2]);
      acc[1][3] = fmaf(a.y, b.w, acc[1][3]);
    }
    __syncthreads();
  }
  float* C = p.C + static_cast<long long>(blockIdx.z) * p.slot_stride;
  const int gn = n0 + tx * 4;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int gm = m0 + ty * 2 + i;
    if (gm >= p.M || gn >= p.N) continue;
    const float4 v = make_float4(apply_act_precise(acc[i][0], p.act), apply_act_precise(acc[i][1], p.act),
                                 apply_act_precise(acc[i][2], p.act), apply_act_precise(acc[i][3], p.act));
    *reinterpret_cast<float4*>(C + static_cast<long long>(gm) * p.ldc + gn) = v;
  }
}

}  // namespace tp
