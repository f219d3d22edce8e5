// Shard reduce + residual + LayerNorm, one CTA per row:
//
//   Z = X + sum_p P_p ;   Y = (Z - mean(Z)) / sqrt(var(Z) + eps) * gamma + beta
//
// The fusion the pages suggest: fold the reduction of the per-shard partial
// sums into the residual add and the next LayerNorm's statistics ("TP到底在切
// 什么" §2.3 and §5.3).  The row statistics are taken over the whole hidden
// row in a fixed order (two passes over registers: mean, then the biased
// variance of the centred values), so a run is bitwise repeatable.
//
// Memory access: every thread moves 8 consecutive elements per step with
// 128-bit loads/stores (2 x float4 of each f32 partial, one uint4 of bf16 X or
// Y), consecutive threads take consecutive 8-element chunks, so each warp
// touches 1 KiB (f32) / 512 B (bf16) contiguous per step.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace tp {

namespace rln {
constexpr int THREADS = 256;
constexpr int MAX_CHUNKS = 8;  // 8-element chunks per thread: H <= 8 * 8 * 256 = 16384
}

struct ReduceLnArgs {
  int S, H;
  int nparts;                 // number of f32 partial-sum buffers (0 = none)
  const float* parts;         // nparts x [S, H], contiguous, part_stride elements apart
  long long part_stride;
  const void* X;              // [S, H] residual, bf16 or f32
  int x_bf16;
  const float* gamma;         // [H] or null (= 1)
  const float* beta;          // [H] or null (= 0)
  float eps;
  void* Y;                    // [S, H], bf16 or f32
  int y_bf16;
};

__device__ __forceinline__ float block_sum_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();  // `red` may still be read from a previous call
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.0f;
#pragma unroll
  for (int i = 0; i < rln::THREADS / 32; ++i) t += red[i];  // same order in every thread
  return t;
}

__device__ __forceinline__ void load8_bf16(const __nv_bfloat16* src, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ void load8_f32(const float* src, float* v) {
  const float4 a = reinterpret_cast<const float4*>(src)[0];
  const float4 b = reinterpret_cast<const float4*>(src)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <int CHUNKS>
__global__ void __launch_bounds__(rln::THREADS) reduce_residual_ln_kernel(const ReduceLnArgs p) {
  __shared__ float red[rln::THREADS / 32];
  const long long row = blockIdx.x;
  const long long base = row * p.H;
  float v[CHUNKS][8];
  float s = 0.0f;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int col = (c * rln::THREADS + threadIdx.x) * 8;
    if (col < p.H) {
      if (p.x_bf16) load8_bf16(static_cast<const __nv_bfloat16*>(p.X) + base + col, v[c]);
      else load8_f32(static_cast<const float*>(p.X) + base + col, v[c]);
      for (int q = 0; q < p.nparts; ++q) {
        float w[8];
        load8_f32(p.parts + q * p.part_stride + base + col, w);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[c][e] += w[e];
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) s += v[c][e];
    }
  }
  const float mean = block_sum_256(s, red) / static_cast<float>(p.H);
  float s2 = 0.0f;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int col = (c * rln::THREADS + threadIdx.x) * 8;
    if (col < p.H) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = v[c][e] - mean;
        s2 = fmaf(d, d, s2);
      }
    }
  }
  const float var = block_sum_256(s2, red) / static_cast<float>(p.H);
  const float rstd = 1.0f / sqrtf(var + p.eps);
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int col = (c * rln::THREADS + threadIdx.x) * 8;
    if (col < p.H) {
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float g = p.gamma ? p.gamma[col + e] : 1.0f;
        const float b = p.beta ? p.beta[col + e] : 0.0f;
        y[e] = fmaf((v[c][e] - mean) * rstd, g, b);
      }
      if (p.y_bf16) {
        uint4 u;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(y[2], y[3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(y[4], y[5]);
        __nv_bfloat162 h3 = __floats2bfloat162_rn(y[6], y[7]);
        u.x = *reinterpret_cast<uint32_t*>(&h0);
        u.y = *reinterpret_cast<uint32_t*>(&h1);
        u.z = *reinterpret_cast<uint32_t*>(&h2);
        u.w = *reinterpret_cast<uint32_t*>(&h3);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.Y) + base + col) = u;
      } else {
        float4* d = reinterpret_cast<float4*>(static_cast<float*>(p.Y) + base + col);
        d[0] = make_float4(y[0], y[1], y[2], y[3]);
        d[1] = make_float4(y[4], y[5], y[6], y[7]);
      }
    }
  }
}

}  // namespace tp
