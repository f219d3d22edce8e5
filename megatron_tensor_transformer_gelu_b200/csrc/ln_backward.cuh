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

// One row per CTA at a time, CH chunks of 8 per thread (H <= CH * 2048).  The
// CTA's per-column dgamma/dbeta sums live in dynamic shared memory as four
// planes of H / 8 float4 (dgamma elements 0..3 and 4..7 of each chunk, then
// dbeta's), so a thread's read-modify-write of its own chunk is conflict-free.
// The row reduction's scratch is double-buffered by row parity, so one
// barrier per row suffices.
#ifndef TP_LNB_MIN_BLOCKS
#define TP_LNB_MIN_BLOCKS 1  // CTAs per SM the register budget of the 1- and 2-chunk kernels is sized for
#endif
// Elementwise work on f32 pairs (fma/add/mul.rn.f32x2): with the row
// constants folded, x̂ = Z r - mean r and dZ = g r + x̂ (-mean(g x̂) r) +
// (-mean(g) r), two pair instructions each.
using f2x = unsigned long long;

// The two bf16 of a 32-bit word as an f32 pair (low half first).
__device__ __forceinline__ f2x lnb_bf2(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ void lnb_gamma4(const float* gamma, int col, f2x (&gm)[4]) {
  if (gamma) {
    const ulonglong2 ga = __ldg(reinterpret_cast<const ulonglong2*>(gamma + col));
    const ulonglong2 gb = __ldg(reinterpret_cast<const ulonglong2*>(gamma + col) + 1);
    gm[0] = ga.x; gm[1] = ga.y; gm[2] = gb.x; gm[3] = gb.y;
  } else {
    const f2x one = f2_pack(1.0f, 1.0f);
#pragma unroll
    for (int e = 0; e < 4; ++e) gm[e] = one;
  }
}

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
  ulonglong2 var[CH], vbr[CH];
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
        const ulonglong2* vp = reinterpret_cast<const ulonglong2*>(p.V + base + k * 8);
        var[c] = __ldcs(vp);
        vbr[c] = __ldcs(vp + 1);
      }
    }
  };
  if (static_cast<int>(blockIdx.x) < p.S) load_row(blockIdx.x);
  int parity = 0;
  for (int row = blockIdx.x; row < p.S; row += gridDim.x, parity ^= 1) {
    const long long base = static_cast<long long>(row) * p.H;
    const f2x r2 = f2_pack(str.y, str.y);
    const f2x b2 = f2_pack(-str.x * str.y, -str.x * str.y);
    f2x xh[CH][4];
    uint4 dyp[CH];
    f2x sg2 = 0ull, sgx2 = 0ull;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int k = c * lnb::THREADS + tid;
      if (k < nch) {
        f2x gm[4];
        lnb_gamma4(p.gamma, k * 8, gm);
        dyp[c] = dyr[c];
        const uint32_t xw[4] = {xr[c].x, xr[c].y, xr[c].z, xr[c].w};
        const uint32_t dw[4] = {dyp[c].x, dyp[c].y, dyp[c].z, dyp[c].w};
        const f2x v[4] = {var[c].x, var[c].y, vbr[c].x, vbr[c].y};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // Z = X + V added as the forward's LayerNorm added it
          xh[c][e] = f2_fma(f2_add(lnb_bf2(xw[e]), v[e]), r2, b2);
          const f2x g = f2_mul(lnb_bf2(dw[e]), gm[e]);
          sg2 = f2_add(sg2, g);
          sgx2 = f2_fma(g, xh[c][e], sgx2);
        }
      }
    }
    if (row + static_cast<int>(gridDim.x) < p.S) load_row(row + gridDim.x);
    float sg, sgx;
    {
      float a0, a1;
      f2_unpack(sg2, a0, a1);
      sg = a0 + a1;
      f2_unpack(sgx2, a0, a1);
      sgx = a0 + a1;
    }
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
    const float c1 = -(tg * inv_h) * str.y, c2 = -(tgx * inv_h) * str.y;
    const f2x c1p = f2_pack(c1, c1), c2p = f2_pack(c2, c2);
    const f2x rr2 = r2;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int k = c * lnb::THREADS + tid;
      if (k < nch) {
        f2x gm[4];
        lnb_gamma4(p.gamma, k * 8, gm);
        const uint32_t dw[4] = {dyp[c].x, dyp[c].y, dyp[c].z, dyp[c].w};
        uint32_t w[4];
        ulonglong2* a = reinterpret_cast<ulonglong2*>(lnb_acc + k);
        ulonglong2 d0 = a[0], d1 = a[nch], e0 = a[2 * nch], e1 = a[3 * nch];
        f2x dg[4] = {d0.x, d0.y, d1.x, d1.y}, db[4] = {e0.x, e0.y, e1.x, e1.y};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const f2x dy = lnb_bf2(dw[e]);
          const f2x dz = f2_fma(xh[c][e], c2p, f2_fma(f2_mul(dy, gm[e]), rr2, c1p));
          float o0, o1;
          f2_unpack(dz, o0, o1);
          __nv_bfloat162 hh = __floats2bfloat162_rn(o0, o1);
          w[e] = *reinterpret_cast<uint32_t*>(&hh);
          dg[e] = f2_fma(dy, xh[c][e], dg[e]);
          db[e] = f2_add(db[e], dy);
        }
        *reinterpret_cast<uint4*>(p.dZ + base + k * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        a[0] = make_ulonglong2(dg[0], dg[1]);
        a[nch] = make_ulonglong2(dg[2], dg[3]);
        a[2 * nch] = make_ulonglong2(db[0], db[1]);
        a[3 * nch] = make_ulonglong2(db[2], db[3]);
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
