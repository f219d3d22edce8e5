// Elementwise steps of the attention backward, per head h (a launch covers a
// group of heads), between GEMMs that run on the tensor cores:
//
//   D_h[r]   = sum_c dO[r, h d + c] * O[r, h d + c]              (rowdot_kernel)
//   P[r, k]  = 2^(S[r, k] * scale_log2 - lse2_h[r])              (softmax_rebuild_kernel)
//   dS[r, k] = P[r, k] * (dP[r, k] - D_h[r]) * scale             (softmax_backward_kernel)
//
// S = Q_h K_h^T (raw scores) and dP = dO_h V_h^T come from GEMMs; lse2 is the
// log2 softmax denominator the forward kept, so P is the forward's softmax of
// the scaled scores.  dS is the softmax's backward (the row projection of dP
// onto P, with sum_k P dP = sum_c dO O = D), scaled by 1/sqrt(d) so that
// dQ = dS K and dK = dS^T Q.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace tp {

// One warp per (row, head): 128 products, 4 per lane (d = 128).
__global__ void __launch_bounds__(256) rowdot_kernel(const __nv_bfloat16* dO, const __nv_bfloat16* O, float* D,
                                                     int S, int H, int nh) {
  griddep_wait();
  griddep_launch_dependents();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= S * nh) return;
  const int h = warp / S, r = warp % S;
  const long long off = static_cast<long long>(r) * H + h * 128 + lane * 4;
  const uint2 a = *reinterpret_cast<const uint2*>(dO + off);
  const uint2 b = *reinterpret_cast<const uint2*>(O + off);
  const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
  float v = 0.0f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float2 x = __bfloat1622float2(a2[i]), y = __bfloat1622float2(b2[i]);
    v = fmaf(x.x, y.x, fmaf(x.y, y.y, v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) D[static_cast<long long>(h) * S + r] = v;
}

// 8 consecutive elements of a [rows, S] matrix per thread (S % 8 == 0),
// grid-stride.  rows = g S for a group of g heads stored one [S, S] matrix
// after another; their per-row vectors (lse2, D) are then consecutive too.
__global__ void __launch_bounds__(256) softmax_rebuild_kernel(const float* Sc, const float* lse2, float scale_log2,
                                                              __nv_bfloat16* P, int rows, int S) {
  griddep_wait();
  griddep_launch_dependents();
  const long long n8 = static_cast<long long>(rows) * S / 8;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long e = i * 8;
    const float m = lse2[e / S];
    const float4 a = __ldcs(reinterpret_cast<const float4*>(Sc + e));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(Sc + e) + 1);
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 h2 = __floats2bfloat162_rn(exp2f(fmaf(v[2 * k], scale_log2, -m)),
                                                exp2f(fmaf(v[2 * k + 1], scale_log2, -m)));
      w[k] = *reinterpret_cast<uint32_t*>(&h2);
    }
    *reinterpret_cast<uint4*>(P + e) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

__global__ void __launch_bounds__(256) softmax_backward_kernel(const __nv_bfloat16* P, const float* dP, const float* D,
                                                               float scale, __nv_bfloat16* dS, int rows, int S) {
  griddep_wait();
  griddep_launch_dependents();
  const long long n8 = static_cast<long long>(rows) * S / 8;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long e = i * 8;
    const float dr = D[e / S];
    const uint4 pw = *reinterpret_cast<const uint4*>(P + e);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&pw);
    const float4 a = __ldcs(reinterpret_cast<const float4*>(dP + e));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(dP + e) + 1);
    const float g[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 p = __bfloat1622float2(p2[k]);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(p.x * (g[2 * k] - dr) * scale, p.y * (g[2 * k + 1] - dr) * scale);
      w[k] = *reinterpret_cast<uint32_t*>(&h2);
    }
    *reinterpret_cast<uint4*>(dS + e) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace tp
