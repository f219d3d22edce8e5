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

// One warp per ROWDOT_ITEMS consecutive (row, head) items (item w = h S + r):
// 128 products per item, 4 per lane (d = 128).  Every item's loads are issued
// before the first product, so a lane has ROWDOT_ITEMS x 16 bytes in flight
// and the grid is ROWDOT_ITEMS times smaller than one item per warp.
constexpr int ROWDOT_ITEMS = 8;
__global__ void __launch_bounds__(256) rowdot_kernel(const __nv_bfloat16* dO, const __nv_bfloat16* O, float* D,
                                                     int S, int H, int nh) {
  griddep_wait();
  griddep_launch_dependents();
  // S * nh fits an int (S <= 2^20 rows, nh <= 128 heads of 128 columns).
  const int warp = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  const int items = S * nh;
  const int w0 = warp * ROWDOT_ITEMS;
  // Item w0's head and row, then the next rows of that head (S >= 128 > the
  // item count, so the row wraps into the next head at most once).
  const int h0 = w0 / S, r0 = w0 - h0 * S;
  uint2 a[ROWDOT_ITEMS], b[ROWDOT_ITEMS];
#pragma unroll
  for (int i = 0; i < ROWDOT_ITEMS; ++i) {
    if (w0 + i < items) {
      const int wrap = r0 + i >= S ? 1 : 0;
      const int h = h0 + wrap, r = r0 + i - wrap * S;
      const long long off = static_cast<long long>(r) * H + h * 128 + lane * 4;
      a[i] = *reinterpret_cast<const uint2*>(dO + off);
      b[i] = *reinterpret_cast<const uint2*>(O + off);
    }
  }
#pragma unroll
  for (int i = 0; i < ROWDOT_ITEMS; ++i) {
    const int w = w0 + i;
    if (w >= items) break;
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a[i]);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b[i]);
    float v = 0.0f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float2 x = __bfloat1622float2(a2[k]), y = __bfloat1622float2(b2[k]);
      v = fmaf(x.x, y.x, fmaf(x.y, y.y, v));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) D[w] = v;
  }
}

}  // namespace tp
