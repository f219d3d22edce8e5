// Backward of the fused residual + LayerNorm, one row per CTA at a time:
//
//   forward   Z = X + sum_p V_p ;  Y = (Z - mean) * r * gamma + beta,  r = 1/sqrt(var + eps)
//   backward  xh = (Z - mean) * r ;  g = dY * gamma
//             dZ = r * (g - mean(g) - xh * mean(g * xh))
//             dgamma = sum over rows of dY * xh ;  dbeta = sum over rows of dY
//
// Z and its statistics are recomputed from the forward's inputs (X and the f32
// partial sums the row-split GEMM left), so the forward keeps no extra tensor.
// The gradient of the weights of each shard stays with its shard
// ("TP到底在切什么" §4); dgamma/dbeta are reduced over rows in a fixed order:
// every CTA accumulates its rows' contributions per column in registers and
// writes one partial row, and a second kernel adds the partial rows.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace tp {

namespace lnb {
constexpr int MAX_WARPS = 16;
}

struct LnBackArgs {
  int S, H;
  int nparts;
  const float* parts;          // nparts x [S, H] f32, part_stride apart
  long long part_stride;
  const __nv_bfloat16* X;      // [S, H]
  const __nv_bfloat16* dY;     // [S, H]
  const float* gamma;          // [H] or null (= 1)
  float eps;
  __nv_bfloat16* dZ;           // [S, H]
  float* partial;              // [gridDim.x][2][H]: per-CTA (dgamma, dbeta) sums
};

// Sum of v over the CTA (all threads get it), fixed order: warp shuffles, then
// the warps' sums in warp order.
__device__ __forceinline__ float lnb_block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __syncthreads();  // red may still be read from the previous reduction
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  __syncthreads();
  float t = 0.0f;
  for (int w = 0; w < nw; ++w) t += red[w];
  return t;
}

// CH chunks of 8 consecutive elements per thread (CH = 1..4, up to 512
// threads, so H <= 16384); chunk c of thread i covers elements
// (c * blockDim.x + i) * 8 ...; chunks past H are masked.  A row takes two
// CTA reductions: (sum z, sum g, sum g z), then sum (z - mean)^2, using
// sum g xh = r (sum g z - mean sum g).  dY is read again (from cache) in the
// last pass instead of being held, to keep registers for Z and the running
// dgamma/dbeta column sums.
__device__ __forceinline__ void lnb_load8_bf16(const __nv_bfloat16* src, float (&v)[8]) {
  const uint4 w = *reinterpret_cast<const uint4*>(src);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    v[2 * e] = f.x;
    v[2 * e + 1] = f.y;
  }
}

// Sum of three values over the CTA (fixed order), as lnb_block_sum.
__device__ __forceinline__ void lnb_block_sum3(float& a, float& b, float& c, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
    c += __shfl_xor_sync(0xffffffffu, c, o);
  }
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) {
    red[warp] = a;
    red[lnb::MAX_WARPS + warp] = b;
    red[2 * lnb::MAX_WARPS + warp] = c;
  }
  __syncthreads();
  float ta = 0.0f, tb = 0.0f, tc = 0.0f;
  for (int w = 0; w < nw; ++w) {
    ta += red[w];
    tb += red[lnb::MAX_WARPS + w];
    tc += red[2 * lnb::MAX_WARPS + w];
  }
  a = ta;
  b = tb;
  c = tc;
}

template <int CH>
__global__ void __launch_bounds__(512) ln_backward_kernel(const LnBackArgs p) {
  __shared__ float red[3 * lnb::MAX_WARPS];
  griddep_wait();  // V and dY come from preceding kernels
  griddep_launch_dependents();
  const int nthr = blockDim.x;
  float z[CH][8], dg[CH][8], db[CH][8];
#pragma unroll
  for (int c = 0; c < CH; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) dg[c][e] = db[c][e] = 0.0f;
  const float inv_h = 1.0f / static_cast<float>(p.H);

  for (int row = blockIdx.x; row < p.S; row += gridDim.x) {
    const long long base = static_cast<long long>(row) * p.H;
    float sz = 0.0f, sg = 0.0f, sgz = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (c * nthr + threadIdx.x) * 8;
      if (col < p.H) {
        float dy[8];
        lnb_load8_bf16(p.X + base + col, z[c]);
        lnb_load8_bf16(p.dY + base + col, dy);
        for (int q = 0; q < p.nparts; ++q) {
          const float4* pp = reinterpret_cast<const float4*>(p.parts + q * p.part_stride + base + col);
          const float4 a = __ldcs(pp), b = __ldcs(pp + 1);
          z[c][0] += a.x; z[c][1] += a.y; z[c][2] += a.z; z[c][3] += a.w;
          z[c][4] += b.x; z[c][5] += b.y; z[c][6] += b.z; z[c][7] += b.w;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float g = p.gamma ? dy[e] * __ldg(p.gamma + col + e) : dy[e];
          sz += z[c][e];
          sg += g;
          sgz = fmaf(g, z[c][e], sgz);
        }
      }
    }
    lnb_block_sum3(sz, sg, sgz, red);
    const float mean = sz * inv_h;
    float v = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (c * nthr + threadIdx.x) * 8;
      if (col < p.H) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float d = z[c][e] - mean;
          v = fmaf(d, d, v);
        }
      }
    }
    const float var = lnb_block_sum(v, red) * inv_h;
    const float r = rsqrtf(var + p.eps);
    const float mg = sg * inv_h;
    const float mgx = r * (sgz - mean * sg) * inv_h;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (c * nthr + threadIdx.x) * 8;
      if (col < p.H) {
        float dy[8];
        lnb_load8_bf16(p.dY + base + col, dy);
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float o[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int i = 2 * e + k;
            const float xh = (z[c][i] - mean) * r;
            const float g = p.gamma ? dy[i] * __ldg(p.gamma + col + i) : dy[i];
            o[k] = r * (g - mg - xh * mgx);
            dg[c][i] = fmaf(dy[i], xh, dg[c][i]);
            db[c][i] += dy[i];
          }
          __nv_bfloat162 h = __floats2bfloat162_rn(o[0], o[1]);
          w[e] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p.dZ + base + col) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  // This CTA's per-column partial sums (zero where it had no rows).
  float* out = p.partial + static_cast<long long>(blockIdx.x) * 2 * p.H;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int col = (c * nthr + threadIdx.x) * 8;
    if (col < p.H) {
      float4* og = reinterpret_cast<float4*>(out + col);
      float4* ob = reinterpret_cast<float4*>(out + p.H + col);
      og[0] = make_float4(dg[c][0], dg[c][1], dg[c][2], dg[c][3]);
      og[1] = make_float4(dg[c][4], dg[c][5], dg[c][6], dg[c][7]);
      ob[0] = make_float4(db[c][0], db[c][1], db[c][2], db[c][3]);
      ob[1] = make_float4(db[c][4], db[c][5], db[c][6], db[c][7]);
    }
  }
}

// The same backward with each row's inputs (X, dY and the f32 partial sums)
// brought into shared memory by untiled bulk copies, issued by one thread
// nst - 1 rows ahead of the row the CTA works on, so that several rows per
// CTA are in flight from HBM while the CTA runs a row's reductions.  256
// threads; thread i's chunk c covers columns (c * 256 + i) * 8 .. + 7.  The
// stage of row i - 1 is refilled (with row i - 1 + nst) once every thread has
// passed row i's first barrier.  Statistics in the same fixed order as the
// register kernel's (warp shuffles, then the warps in order).
// Stage layout: [X row bf16][dY row bf16][partial rows f32 ...].
namespace lnbb {
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
}

__device__ __forceinline__ void lnbb_issue_row(const LnBackArgs& p, long long row, uint8_t* dst, uint64_t* bar) {
  const uint32_t hb = static_cast<uint32_t>(p.H) * 2u, fb = static_cast<uint32_t>(p.H) * 4u;
  mbar_arrive_expect_tx(bar, 2 * hb + static_cast<uint32_t>(p.nparts) * fb);
  bulk_load_1d(dst, p.X + row * p.H, hb, bar);
  bulk_load_1d(dst + hb, p.dY + row * p.H, hb, bar);
  for (int q = 0; q < p.nparts; ++q) bulk_load_1d(dst + 2 * hb + q * fb, p.parts + q * p.part_stride + row * p.H, fb, bar);
}

__device__ __forceinline__ void lnbb_load8(const uint8_t* src_bf16, float (&v)[8]) {
  const uint4 w = *reinterpret_cast<const uint4*>(src_bf16);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    v[2 * e] = f.x;
    v[2 * e + 1] = f.y;
  }
}

template <int CH>
__global__ void __launch_bounds__(lnbb::THREADS) ln_backward_bulk_kernel(const LnBackArgs p, int nst, int stage_bytes) {
  extern __shared__ __align__(128) uint8_t lnbb_smem[];
  __shared__ uint64_t full[4];
  __shared__ float red[2][4][lnbb::WARPS];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t hb = static_cast<uint32_t>(p.H) * 2u, fb = static_cast<uint32_t>(p.H) * 4u;
  if (tid == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
  }
  __syncthreads();
  griddep_wait();  // V and dY come from preceding kernels
  griddep_launch_dependents();
  float dg[CH][8], db[CH][8];
#pragma unroll
  for (int c = 0; c < CH; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) dg[c][e] = db[c][e] = 0.0f;
  const float inv_h = 1.0f / static_cast<float>(p.H);
  const int n_my = blockIdx.x < p.S ? (p.S - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1 : 0;
  int issued = 0;
  if (tid == 0) {
    for (; issued < nst && issued < n_my; ++issued)
      lnbb_issue_row(p, blockIdx.x + static_cast<long long>(issued) * gridDim.x, lnbb_smem + issued * stage_bytes,
                     &full[issued]);
  }
  int i = 0;
  for (; i < n_my; ++i) {
    const int s = i % nst;
    const long long row = blockIdx.x + static_cast<long long>(i) * gridDim.x;
    const uint8_t* st = lnbb_smem + s * stage_bytes;
    const bool ok = mbar_wait(&full[s], static_cast<uint32_t>((i / nst) & 1));
    if (!__syncthreads_and(ok)) break;
    float z[CH][8];
    float sz = 0.0f, sg = 0.0f, sgz = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (c * lnbb::THREADS + tid) * 8;
      if (col < p.H) {
        float dy[8], gm[8];
        lnbb_load8(st + col * 2, z[c]);
        lnbb_load8(st + hb + col * 2, dy);
        for (int q = 0; q < p.nparts; ++q) {
          const float4* pp = reinterpret_cast<const float4*>(st + 2 * hb + q * fb + col * 4);
          const float4 a = pp[0], b = pp[1];
          z[c][0] += a.x; z[c][1] += a.y; z[c][2] += a.z; z[c][3] += a.w;
          z[c][4] += b.x; z[c][5] += b.y; z[c][6] += b.z; z[c][7] += b.w;
        }
        if (p.gamma) {
          const float4 a = __ldg(reinterpret_cast<const float4*>(p.gamma + col));
          const float4 b = __ldg(reinterpret_cast<const float4*>(p.gamma + col) + 1);
          gm[0] = a.x; gm[1] = a.y; gm[2] = a.z; gm[3] = a.w; gm[4] = b.x; gm[5] = b.y; gm[6] = b.z; gm[7] = b.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) gm[e] = 1.0f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float g = dy[e] * gm[e];
          sz += z[c][e];
          sg += g;
          sgz = fmaf(g, z[c][e], sgz);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sz += __shfl_xor_sync(0xffffffffu, sz, o);
      sg += __shfl_xor_sync(0xffffffffu, sg, o);
      sgz += __shfl_xor_sync(0xffffffffu, sgz, o);
    }
    if (lane == 0) {
      red[i & 1][0][warp] = sz;
      red[i & 1][1][warp] = sg;
      red[i & 1][2][warp] = sgz;
    }
    __syncthreads();
    // Every thread is past row i - 1: its stage takes the row nst - 1 ahead.
    if (tid == 0 && i > 0 && issued < n_my) {
      fence_proxy_async_smem();
      const int sp = (i - 1) % nst;
      lnbb_issue_row(p, blockIdx.x + static_cast<long long>(issued) * gridDim.x, lnbb_smem + sp * stage_bytes,
                     &full[sp]);
      ++issued;
    }
    float tz = 0.0f, tg = 0.0f, tgz = 0.0f;
#pragma unroll
    for (int w = 0; w < lnbb::WARPS; ++w) {
      tz += red[i & 1][0][w];
      tg += red[i & 1][1][w];
      tgz += red[i & 1][2][w];
    }
    const float mean = tz * inv_h;
    float v = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      if ((c * lnbb::THREADS + tid) * 8 < p.H) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float d = z[c][e] - mean;
          v = fmaf(d, d, v);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[i & 1][3][warp] = v;
    __syncthreads();
    float tv = 0.0f;
#pragma unroll
    for (int w = 0; w < lnbb::WARPS; ++w) tv += red[i & 1][3][w];
    const float r = rsqrtf(tv * inv_h + p.eps);
    const float mg = tg * inv_h;
    const float mgx = r * (tgz - mean * tg) * inv_h;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (c * lnbb::THREADS + tid) * 8;
      if (col < p.H) {
        float dy[8], gm[8];
        lnbb_load8(st + hb + col * 2, dy);
        if (p.gamma) {
          const float4 a = __ldg(reinterpret_cast<const float4*>(p.gamma + col));
          const float4 b = __ldg(reinterpret_cast<const float4*>(p.gamma + col) + 1);
          gm[0] = a.x; gm[1] = a.y; gm[2] = a.z; gm[3] = a.w; gm[4] = b.x; gm[5] = b.y; gm[6] = b.z; gm[7] = b.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) gm[e] = 1.0f;
        }
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float o[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int j = 2 * e + k;
            const float xh = (z[c][j] - mean) * r;
            o[k] = r * (dy[j] * gm[j] - mg - xh * mgx);
            dg[c][j] = fmaf(dy[j], xh, dg[c][j]);
            db[c][j] += dy[j];
          }
          __nv_bfloat162 h = __floats2bfloat162_rn(o[0], o[1]);
          w[e] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p.dZ + row * p.H + col) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  // After an error exit, copies issued but not consumed must land (bounded)
  // before the CTA's shared memory is released.
  if (tid == 0) {
    for (int j = i; j < issued; ++j) {
      const uint32_t a = smem_u32(&full[j % nst]);
      const long long t0 = clock64();
      while (!mbar_try_wait(a, static_cast<uint32_t>((j / nst) & 1)) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
    }
  }
  // This CTA's per-column partial sums (zero where it had no rows).
  float* out = p.partial + static_cast<long long>(blockIdx.x) * 2 * p.H;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int col = (c * lnbb::THREADS + tid) * 8;
    if (col < p.H) {
      float4* og = reinterpret_cast<float4*>(out + col);
      float4* ob = reinterpret_cast<float4*>(out + p.H + col);
      og[0] = make_float4(dg[c][0], dg[c][1], dg[c][2], dg[c][3]);
      og[1] = make_float4(dg[c][4], dg[c][5], dg[c][6], dg[c][7]);
      ob[0] = make_float4(db[c][0], db[c][1], db[c][2], db[c][3]);
      ob[1] = make_float4(db[c][4], db[c][5], db[c][6], db[c][7]);
    }
  }
}

// dgamma[j] = sum_b partial[b][0][j], dbeta[j] = sum_b partial[b][1][j].
// A CTA takes 32 columns with 32 warps: warp w sums the partial rows
// b = w, w + 32, ... (each load a 128-byte row segment, four rows in flight
// in separate accumulators added in a fixed order), then warp 0 adds the 32
// warps' sums in warp order, so the result is deterministic.
constexpr int LNB_PARAM_SLICES = 32;
__global__ void __launch_bounds__(32 * LNB_PARAM_SLICES)
    ln_grad_params_kernel(const float* partial, int nblk, int H, float* dgamma, float* dbeta) {
  __shared__ float sa[LNB_PARAM_SLICES][33], sb[LNB_PARAM_SLICES][33];
  const int lane = threadIdx.x & 31, slice = threadIdx.x >> 5;
  griddep_wait();  // the partial rows come from the preceding kernel
  griddep_launch_dependents();
  const int j = blockIdx.x * 32 + lane;
  float a[4] = {0.0f, 0.0f, 0.0f, 0.0f}, b[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if (j < H) {
    const long long step = 2LL * H;
    int k = slice;
    for (; k + 3 * LNB_PARAM_SLICES < nblk; k += 4 * LNB_PARAM_SLICES) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
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
  sa[slice][lane] = (a[0] + a[1]) + (a[2] + a[3]);
  sb[slice][lane] = (b[0] + b[1]) + (b[2] + b[3]);
  __syncthreads();
  if (slice == 0 && j < H) {
    float ta = 0.0f, tb = 0.0f;
#pragma unroll 8
    for (int w = 0; w < LNB_PARAM_SLICES; ++w) {
      ta += sa[w][lane];
      tb += sb[w][lane];
    }
    if (dgamma) dgamma[j] = ta;
    if (dbeta) dbeta[j] = tb;
  }
}

}  // namespace tp
