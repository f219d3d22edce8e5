// Row dots of the attention backward, per head h:
//
//   D_h[r] = sum_c dO[r, h d + c] * O[r, h d + c]
//
// Since O_h = P_h V_h, D_h[r] = sum_k P_h[r, k] dP_h[r, k] with dP_h = dO_h V_h^T:
// the term the softmax's backward subtracts from every dP_h[r, k] before
// multiplying by P_h[r, k], dS_h = P_h (dP_h - D_h) / sqrt d.  That product is
// taken in the epilogue of the GEMM that makes dP_h, and P_h itself,
// 2^(S_h scale_log2 - lse2_h), in the epilogue of the GEMM that makes the
// scores S_h = Q_h K_h^T (lse2 being the log2 softmax denominator the forward
// kept).
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

}  // namespace tp
