// Backward of the fused residual + LayerNorm:
//
//   forward   Z = X + V ;  Y = (Z - mean) * r * gamma + beta,  r = 1/sqrt(var + eps)
//   backward  xh = (Z - mean) * r ;  g = dY * gamma
//             dZ = r * (g - mean(g) - xh * mean(g * xh))
//             dgamma = sum over rows of dY * xh ;  dbeta = sum over rows of dY
//
// Z is recomputed from the forward's inputs (X and the f32 sum V the
// row-split GEMM left) with the forward's own row statistics (mean, r),
// which the training forward's LayerNorm stored: the same values the forward
// normalised with, and one CTA reduction per row (sum g, sum g xh) instead
// of the three a recomputation of the statistics takes.  The gradient of the
// weights of each shard stays with its shard ("TP到底在切什么" §4);
// dgamma/dbeta are reduced over rows in a fixed order: every CTA adds its
// rows' contributions per column into shared memory (each thread owns its
// columns) and writes one partial row, and a second kernel adds the partial
// rows.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace tp {

namespace lnb {
constexpr int THREADS = 256;  // 8 warps; thread i's chunk c covers columns (c * 256 + i) * 8 .. + 7
constexpr int WARPS = THREADS / 32;
constexpr int MAX_CH = 8;     // H <= 16384
}

struct LnBackArgs {
  int S, H;
  const float* V;              // [S, H] f32: the row-split GEMM's output (Z = X + V)
  const float* stats;          // [S][2] f32: the forward's (mean, r) of each row
  const __nv_bfloat16* X;      // [S, H]
  const __nv_bfloat16* dY;     // [S, H]
  const float* gamma;          // [H] or null (= 1)
  __nv_bfloat16* dZ;           // [S, H]
  float* partial;              // [gridDim.x][2][H]: per-CTA (dgamma, dbeta) sums
};

__device__ __forceinline__ void lnb_gamma8(const float* gamma, int col, float (&gm)[8]) {
  if (gamma) {
    const float4 ga = __ldg(reinterpret_cast<const float4*>(gamma + col));
    const float4 gb = __ldg(reinterpret_cast<const float4*>(gamma + col) + 1);
    gm[0] = ga.x; gm[1] = ga.y; gm[2] = ga.z; gm[3] = ga.w;
    gm[4] = gb.x; gm[5] = gb.y; gm[6] = gb.z; gm[7] = gb.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) gm[e] = 1.0f;
  }
}

__device__ __forceinline__ void lnb_unpack8(const uint4& w, float (&v)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    v[2 * e] = f.x;
    v[2 * e + 1] = f.y;
  }
}

// One row per CTA at a time, CH chunks of 8 per thread (H <= CH * 2048).  The
// CTA's per-column dgamma/dbeta sums live in dynamic shared memory as four
// planes of H / 8 float4 (dgamma elements 0..3 and 4..7 of each chunk, then
// dbeta's), so a thread's read-modify-write of its own chunk is conflict-free.
// The row reduction's scratch is double-buffered by row parity, so one
// barrier per row suffices.
#ifndef TP_LNB_MIN_BLOCKS
#define TP_LNB_MIN_BLOCKS 1  // CTAs per SM the register budget of the 1- and 2-chunk kernels is sized for
#endif
template <int CH>
__global__ void __launch_bounds__(lnb::THREADS, CH <= 2 ? TP_LNB_MIN_BLOCKS : 1) ln_backward_kernel(const LnBackArgs p) {
  extern __shared__ float4 lnb_acc[];  // [4][H / 8]
  __shared__ float red[2][2][lnb::WARPS];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nch = p.H / 8;  // chunks of the row
  for (int i = tid; i < 4 * nch; i += lnb::THREADS) lnb_acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  griddep_wait();  // V, the statistics and dY come from preceding kernels
  griddep_launch_dependents();
  const float inv_h = 1.0f / static_cast<float>(p.H);
  // The row in flight: its loads are issued one row ahead, before the
  // current row's reduction barrier, so they overlap that row's reduction,
  // its dZ stores and its dgamma/dbeta updates.
  uint4 xr[CH], dyr[CH];
  float4 var[CH], vbr[CH];
  float2 str = make_float2(0.0f, 0.0f);
  auto load_row = [&](int row) {
    const long long base = static_cast<long long>(row) * p.H;
    str = *reinterpret_cast<const float2*>(p.stats + 2LL * row);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int k = c * lnb::THREADS + tid;
      if (k < nch) {
        xr[c] = *reinterpret_cast<const uint4*>(p.X + base + k * 8);
        dyr[c] = *reinterpret_cast<const uint4*>(p.dY + base + k * 8);
        const float4* vp = reinterpret_cast<const float4*>(p.V + base + k * 8);
        var[c] = __ldcs(vp);
        vbr[c] = __ldcs(vp + 1);
      }
    }
  };
  if (static_cast<int>(blockIdx.x) < p.S) load_row(blockIdx.x);
  int parity = 0;
  for (int row = blockIdx.x; row < p.S; row += gridDim.x, parity ^= 1) {
    const long long base = static_cast<long long>(row) * p.H;
    const float2 st = str;
    float xh[CH][8];
    uint4 dyp[CH];
    float sg = 0.0f, sgx = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int k = c * lnb::THREADS + tid;
      if (k < nch) {
        float x[8], dy[8], gm[8];
        lnb_unpack8(xr[c], x);
        dyp[c] = dyr[c];
        const float v[8] = {var[c].x, var[c].y, var[c].z, var[c].w, vbr[c].x, vbr[c].y, vbr[c].z, vbr[c].w};
        lnb_unpack8(dyp[c], dy);
        lnb_gamma8(p.gamma, k * 8, gm);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          // Z = X + V added as the forward's LayerNorm added it
          xh[c][e] = (x[e] + v[e] - st.x) * st.y;
          const float g = dy[e] * gm[e];
          sg += g;
          sgx = fmaf(g, xh[c][e], sgx);
        }
      }
    }
    if (row + static_cast<int>(gridDim.x) < p.S) load_row(row + gridDim.x);
    // Row sums: warp shuffles, then the 8 warps' sums in warp order.
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sg += __shfl_xor_sync(0xffffffffu, sg, o);
      sgx += __shfl_xor_sync(0xffffffffu, sgx, o);
    }
    if (lane == 0) {
      red[parity][0][warp] = sg;
      red[parity][1][warp] = sgx;
    }
    __syncthreads();
    float tg = 0.0f, tgx = 0.0f;
#pragma unroll
    for (int w = 0; w < lnb::WARPS; ++w) {
      tg += red[parity][0][w];
      tgx += red[parity][1][w];
    }
    const float mg = tg * inv_h, mgx = tgx * inv_h;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int k = c * lnb::THREADS + tid;
      if (k < nch) {
        float dy[8], gm[8];
        lnb_unpack8(dyp[c], dy);
        lnb_gamma8(p.gamma, k * 8, gm);
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float o0 = st.y * (dy[2 * e] * gm[2 * e] - mg - xh[c][2 * e] * mgx);
          const float o1 = st.y * (dy[2 * e + 1] * gm[2 * e + 1] - mg - xh[c][2 * e + 1] * mgx);
          __nv_bfloat162 hh = __floats2bfloat162_rn(o0, o1);
          w[e] = *reinterpret_cast<uint32_t*>(&hh);
        }
        *reinterpret_cast<uint4*>(p.dZ + base + k * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        float4* a = lnb_acc + k;
        float4 d0 = a[0], d1 = a[nch], b0 = a[2 * nch], b1 = a[3 * nch];
        d0.x = fmaf(dy[0], xh[c][0], d0.x); d0.y = fmaf(dy[1], xh[c][1], d0.y);
        d0.z = fmaf(dy[2], xh[c][2], d0.z); d0.w = fmaf(dy[3], xh[c][3], d0.w);
        d1.x = fmaf(dy[4], xh[c][4], d1.x); d1.y = fmaf(dy[5], xh[c][5], d1.y);
        d1.z = fmaf(dy[6], xh[c][6], d1.z); d1.w = fmaf(dy[7], xh[c][7], d1.w);
        b0.x += dy[0]; b0.y += dy[1]; b0.z += dy[2]; b0.w += dy[3];
        b1.x += dy[4]; b1.y += dy[5]; b1.z += dy[6]; b1.w += dy[7];
        a[0] = d0;
        a[nch] = d1;
        a[2 * nch] = b0;
        a[3 * nch] = b1;
      }
    }
  }
  // This CTA's per-column partial sums (zero where it had no rows); each
  // thread wrote only its own chunks, so no barrier is needed.
  float* out = p.partial + static_cast<long long>(blockIdx.x) * 2 * p.H;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int k = c * lnb::THREADS + tid;
    if (k < nch) {
      float4* og = reinterpret_cast<float4*>(out + k * 8);
      float4* ob = reinterpret_cast<float4*>(out + p.H + k * 8);
      og[0] = lnb_acc[k];
      og[1] = lnb_acc[nch + k];
      ob[0] = lnb_acc[2 * nch + k];
      ob[1] = lnb_acc[3 * nch + k];
    }
  }
}

// dgamma[j] = sum_b partial[b][0][j], dbeta[j] = sum_b partial[b][1][j].
// A CTA takes 32 columns with 32 warps: warp w sums the partial rows
// b = w, w + 32, ... (each load a 128-byte row segment, eight rows in flight
// in separate accumulators added in a fixed order), then warp 0 adds the 32
// warps' sums in warp order, so the result is deterministic.
constexpr int LNB_PARAM_SLICES = 32;
constexpr int LNB_PARAM_UNROLL = 8;
__global__ void __launch_bounds__(32 * LNB_PARAM_SLICES)
    ln_grad_params_kernel(const float* partial, int nblk, int H, float* dgamma, float* dbeta) {
  __shared__ float sa[LNB_PARAM_SLICES][33], sb[LNB_PARAM_SLICES][33];
  const int lane = threadIdx.x & 31, slice = threadIdx.x >> 5;
  griddep_wait();  // the partial rows come from the preceding kernel
  griddep_launch_dependents();
  const int j = blockIdx.x * 32 + lane;
  float a[LNB_PARAM_UNROLL], b[LNB_PARAM_UNROLL];
#pragma unroll
  for (int u = 0; u < LNB_PARAM_UNROLL; ++u) a[u] = b[u] = 0.0f;
  if (j < H) {
    const long long step = 2LL * H;
    int k = slice;
    for (; k + (LNB_PARAM_UNROLL - 1) * LNB_PARAM_SLICES < nblk; k += LNB_PARAM_UNROLL * LNB_PARAM_SLICES) {
#pragma unroll
      for (int u = 0; u < LNB_PARAM_UNROLL; ++u) {
        const float* row = partial + (k + u * LNB_PARAM_SLICES) * step;
        a[u] += row[j];
        b[u] += row[H + j];
      }
    }
    for (; k < nblk; k += LNB_PARAM_SLICES) {
      a[0] += partial[k * step + j];
      b[0] += partial[k * step + H + j];
    }
  }
  float ta = 0.0f, tb = 0.0f;
#pragma unroll
  for (int u = 0; u < LNB_PARAM_UNROLL; ++u) {
    ta += a[u];
    tb += b[u];
  }
  sa[slice][lane] = ta;
  sb[slice][lane] = tb;
  __syncthreads();
  if (slice == 0 && j < H) {
    float sa_t = 0.0f, sb_t = 0.0f;
#pragma unroll 8
    for (int w = 0; w < LNB_PARAM_SLICES; ++w) {
      sa_t += sa[w][lane];
      sb_t += sb[w][lane];
    }
    if (dgamma) dgamma[j] = sa_t;
    if (dbeta) dbeta[j] = sb_t;
  }
}

}  // namespace tp
