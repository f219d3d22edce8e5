// Shard reduce + residual + LayerNorm, 1 to 8 rows per CTA:
//
//   Z = X + sum_p P_p ;   Y = (Z - mean(Z)) / sqrt(var(Z) + eps) * gamma + beta
//
// The fusion the pages suggest: fold the reduction of the per-shard partial
// sums into the residual add and the next LayerNorm's statistics ("TP到底在切
// 什么" §2.3 and §5.3).  The row statistics are taken over the whole hidden
// row in a fixed order (two passes over registers: mean, then the biased
// variance of the centred values), so a run is bitwise repeatable.
//
// Memory access: every lane moves 8 consecutive elements per chunk with
// 128-bit loads/stores (2 x float4 of each f32 partial, one uint4 of bf16 X or
// Y); consecutive lanes take consecutive chunks, so each warp touches 1 KiB
// (f32) / 512 B (bf16) contiguous per step.  The f32 partials are read once,
// with the streaming (evict-first) cache hint.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace tp {

// Single-partial rows: add each chunk's partial as it arrives (1: fewer live
// registers, five 256-thread CTAs per SM; the forward LayerNorm of the
// 2048 x 4096 MLP measured 17.1-17.4 us against 20.7 us), or load X and the
// partial of every chunk before the first add (0).
#ifndef TP_RLN_LEAN
#define TP_RLN_LEAN 1
#endif

namespace rln {
constexpr int THREADS = 256;       // 8 warps per CTA (up to 8 warps per row)
constexpr int MAX_WPR = 16;        // warps per row (CTAs grow to 16 warps)
constexpr int MAX_CH = 4;          // 8-element chunks per lane
constexpr int MAX_H = MAX_WPR * 32 * MAX_CH * 8;  // 16384
// CTA size for WPR warps per row: 8 warps, or one row of WPR warps.
__host__ __device__ constexpr int cta_threads(int wpr) { return wpr > 8 ? wpr * 32 : THREADS; }
}

constexpr int RLN_MAX_PTRS = 8;  // partial sources / output copies given as pointer lists

struct ReduceLnArgs {
  int S, H;
  int nparts;                 // number of f32 partial-sum buffers (0 = none)
  const float* parts;         // nparts x [S, H], contiguous, part_stride elements apart; or null:
  long long part_stride;
  const float* part_ptr[RLN_MAX_PTRS];  // ... partial q at part_ptr[q] ([S, H] each; on this GPU or,
                                        // through peer access, on another: the reduce-scatter's loads)
  const void* X;              // [S, H] residual, bf16 or f32
  int x_bf16;
  const float* gamma;         // [H] or null (= 1)
  const float* beta;          // [H] or null (= 0)
  float eps;
  void* Y;                    // [S, H], bf16 or f32
  int y_bf16;
  int ny_extra;               // further copies of Y written (the all-gather's stores), 0..RLN_MAX_PTRS-1
  void* y_extra[RLN_MAX_PTRS];
  int apply_ln;               // 0: Y = X + sum_p P_p only (pre-LN residual stream)
  float* stats;               // optional [S][2]: each row's (mean, 1/sqrt(var + eps)), for a backward pass
};

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

// Streaming load (read once: evict first).
__device__ __forceinline__ void load8_f32(const float* src, float* v) {
  const float4 a = __ldcs(reinterpret_cast<const float4*>(src));
  const float4 b = __ldcs(reinterpret_cast<const float4*>(src) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Cached load (gamma/beta are read by every row).
__device__ __forceinline__ void load8_f32_keep(const float* src, float* v) {
  const float4 a = reinterpret_cast<const float4*>(src)[0];
  const float4 b = reinterpret_cast<const float4*>(src)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// 8 consecutive output values, bf16 (one 16-byte store) or f32 (two), into Y
// and into each extra copy.
__device__ __forceinline__ void store8_to(void* Y, int y_bf16, long long off, const uint4& u, const float* y) {
  if (y_bf16) {
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(Y) + off) = u;
  } else {
    float4* d = reinterpret_cast<float4*>(static_cast<float*>(Y) + off);
    d[0] = make_float4(y[0], y[1], y[2], y[3]);
    d[1] = make_float4(y[4], y[5], y[6], y[7]);
  }
}

__device__ __forceinline__ void store8(const ReduceLnArgs& p, long long off, const float* y) {
  uint4 u = make_uint4(0u, 0u, 0u, 0u);
  if (p.y_bf16) {
    __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(y[2], y[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(y[4], y[5]);
    __nv_bfloat162 h3 = __floats2bfloat162_rn(y[6], y[7]);
    u.x = *reinterpret_cast<uint32_t*>(&h0);
    u.y = *reinterpret_cast<uint32_t*>(&h1);
    u.z = *reinterpret_cast<uint32_t*>(&h2);
    u.w = *reinterpret_cast<uint32_t*>(&h3);
  }
  store8_to(p.Y, p.y_bf16, off, u, y);
  for (int o = 0; o < p.ny_extra; ++o) store8_to(p.y_extra[o], p.y_bf16, off, u, y);
}

// One row is handled by WPR consecutive warps; a CTA holds max(1, 8 / WPR)
// rows at a time and walks row groups blockIdx.x, blockIdx.x + gridDim.x, ...
// (the grid is sized to the number of CTAs resident at once, so there is no
// partial last wave).  Lane l of warp w (of the row) owns chunks c = 0..CH-1
// at column ((c * WPR + w) * 32 + l) * 8, so each warp reads 32 consecutive
// 8-element chunks per step.  Few values per lane (CH = 2 up to H = 4096, 4
// beyond) keep registers low and occupancy high; larger H uses more warps per
// row.  NP1 specialises the common single partial so that every load of a row
// is issued before its first add.
#ifndef TP_RLN_CH4_MIN_BLOCKS
#define TP_RLN_CH4_MIN_BLOCKS 4
#endif
template <int WPR, int CH, bool NP1>
__global__ void __launch_bounds__(rln::cta_threads(WPR),
                                  (TP_RLN_LEAN && rln::cta_threads(WPR) == 256) ? (CH <= 2 ? 5 : TP_RLN_CH4_MIN_BLOCKS) : 1)
    reduce_residual_ln_kernel(const ReduceLnArgs p) {
  constexpr int RPC = WPR > 8 ? 1 : rln::THREADS / 32 / WPR;  // rows per CTA
  __shared__ float red[2][RPC][WPR];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rloc = warp / WPR, wr = warp % WPR;
  griddep_wait();  // the partial sums come from the preceding kernel
  griddep_launch_dependents();
  const int groups = (p.S + RPC - 1) / RPC;
  for (int g = blockIdx.x; g < groups; g += gridDim.x) {
    const long long row = static_cast<long long>(g) * RPC + rloc;
    const bool live = row < p.S && rloc < RPC;
    const long long base = row * p.H;
    float v[CH][8];
    if (NP1) {
#if TP_RLN_LEAN
      // each chunk's partial added as it arrives: fewer live registers, more
      // CTAs resident per SM
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int col = ((c * WPR + wr) * 32 + lane) * 8;
        if (live && col < p.H) {
          float w[8];
          if (p.x_bf16) load8_bf16(static_cast<const __nv_bfloat16*>(p.X) + base + col, v[c]);
          else load8_f32(static_cast<const float*>(p.X) + base + col, v[c]);
          load8_f32(p.parts + base + col, w);
#pragma unroll
          for (int e = 0; e < 8; ++e) v[c][e] += w[e];
        }
      }
#else
      float w[CH][8];
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int col = ((c * WPR + wr) * 32 + lane) * 8;
        if (live && col < p.H) {
          if (p.x_bf16) load8_bf16(static_cast<const __nv_bfloat16*>(p.X) + base + col, v[c]);
          else load8_f32(static_cast<const float*>(p.X) + base + col, v[c]);
          load8_f32(p.parts + base + col, w[c]);
        }
      }
#pragma unroll
      for (int c = 0; c < CH; ++c)
#pragma unroll
        for (int e = 0; e < 8; ++e) v[c][e] += w[c][e];
#endif
    } else {
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int col = ((c * WPR + wr) * 32 + lane) * 8;
        if (live && col < p.H) {
          if (p.x_bf16) load8_bf16(static_cast<const __nv_bfloat16*>(p.X) + base + col, v[c]);
          else load8_f32(static_cast<const float*>(p.X) + base + col, v[c]);
        }
      }
      for (int q = 0; q < p.nparts; ++q) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const int col = ((c * WPR + wr) * 32 + lane) * 8;
          if (live && col < p.H) {
            float w[8];
            const float* src = p.parts ? p.parts + q * p.part_stride : p.part_ptr[q];
            load8_f32(src + base + col, w);
#pragma unroll
            for (int e = 0; e < 8; ++e) v[c][e] += w[e];
          }
        }
      }
    }
    if (!p.apply_ln) {
      // residual add only: Y = X + sum of the partials
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int col = ((c * WPR + wr) * 32 + lane) * 8;
        if (live && col < p.H) store8(p, base + col, v[c]);
      }
      continue;  // no shared memory touched: no barrier needed
    }
    float s = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = ((c * WPR + wr) * 32 + lane) * 8;
      if (live && col < p.H) {
#pragma unroll
        for (int e = 0; e < 8; ++e) s += v[c][e];
      }
    }
    // mean over the row: warp shuffle, then the row's WPR warps in fixed order
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0 && rloc < RPC) red[0][rloc][wr] = s;
    __syncthreads();
    float tot = 0.0f;
    if (rloc < RPC) {
#pragma unroll
      for (int i = 0; i < WPR; ++i) tot += red[0][rloc][i];
    }
    const float mean = tot / static_cast<float>(p.H);
    float s2 = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = ((c * WPR + wr) * 32 + lane) * 8;
      if (live && col < p.H) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float d = v[c][e] - mean;
          s2 = fmaf(d, d, s2);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    if (lane == 0 && rloc < RPC) red[1][rloc][wr] = s2;
    __syncthreads();
    float tot2 = 0.0f;
    if (rloc < RPC) {
#pragma unroll
      for (int i = 0; i < WPR; ++i) tot2 += red[1][rloc][i];
    }
    const float var = tot2 / static_cast<float>(p.H);
    const float rstd = 1.0f / sqrtf(var + p.eps);
    if (p.stats && live && wr == 0 && lane == 0)
      *reinterpret_cast<float2*>(p.stats + 2 * row) = make_float2(mean, rstd);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = ((c * WPR + wr) * 32 + lane) * 8;
      if (live && col < p.H) {
        float gm[8], bt[8];
        if (p.gamma) load8_f32_keep(p.gamma + col, gm);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) gm[e] = 1.0f;
        }
        if (p.beta) load8_f32_keep(p.beta + col, bt);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) bt[e] = 0.0f;
        }
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = fmaf((v[c][e] - mean) * rstd, gm[e], bt[e]);
        store8(p, base + col, y);
      }
    }
    __syncthreads();  // `red` is reused by the next row group
  }
}

// ---------------------------------------- rows loaded one group ahead (bf16 X)
// The common case of the sublayers (one partial, bf16 X, the LN applied; Y
// bf16 or f32) with the row-group walk of the kernel above, plus two things:
//  - each thread issues the loads of its next row group before the current
//    group's two block reductions, so they overlap the barriers and stores;
//  - the elementwise work runs on f32 pairs (add/sub/mul/fma.rn.f32x2):
//    Z = X + P, the row sum, the centred squares and
//    Y = (Z - mean) (r gamma) + beta take one or two pair instructions per
//    two elements.
// The statistics keep the two-pass form (mean, then the mean square of
// Z - mean), reduced by warp shuffles and then across the row's warps in warp
// order, so results are repeatable.
#ifndef TP_RLN_PF_MIN_BLOCKS
#define TP_RLN_PF_MIN_BLOCKS 4  // CTAs per SM the two-chunk kernel's registers are sized for
#endif
using rln_f2 = unsigned long long;

__device__ __forceinline__ rln_f2 rln_bf2(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <int WPR, int CH>
__global__ void __launch_bounds__(rln::cta_threads(WPR), CH <= 2 ? TP_RLN_PF_MIN_BLOCKS : 2)
    reduce_residual_ln_pf2_kernel(const ReduceLnArgs p) {
  constexpr int RPC = WPR > 8 ? 1 : rln::THREADS / 32 / WPR;  // rows per CTA
  __shared__ float red[2][RPC][WPR];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rloc = warp / WPR, wr = warp % WPR;
  griddep_wait();  // the partial sums come from the preceding kernel
  griddep_launch_dependents();
  const int groups = (p.S + RPC - 1) / RPC;
  uint4 xr[CH];
  ulonglong2 pra[CH], prb[CH];
  auto prefetch = [&](int gg) {
    const long long prow = static_cast<long long>(gg) * RPC + rloc;
    const bool plive = gg < groups && prow < p.S && rloc < RPC;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = ((c * WPR + wr) * 32 + lane) * 8;
      if (plive && col < p.H) {
        xr[c] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.X) + prow * p.H + col);
        const ulonglong2* src = reinterpret_cast<const ulonglong2*>(p.parts + prow * p.H + col);
        pra[c] = __ldcs(src);
        prb[c] = __ldcs(src + 1);
      }
    }
  };
  prefetch(blockIdx.x);
  const float inv_h = 1.0f / static_cast<float>(p.H);
  for (int g = blockIdx.x; g < groups; g += gridDim.x) {
    const long long row = static_cast<long long>(g) * RPC + rloc;
    const bool live = row < p.S && rloc < RPC;
    const long long base = row * p.H;
    rln_f2 v[CH][4];
    rln_f2 sum2 = 0ull;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = ((c * WPR + wr) * 32 + lane) * 8;
      if (live && col < p.H) {
        const uint32_t xw[4] = {xr[c].x, xr[c].y, xr[c].z, xr[c].w};
        const rln_f2 pw[4] = {pra[c].x, pra[c].y, prb[c].x, prb[c].y};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[c][e] = f2_add(rln_bf2(xw[e]), pw[e]);
          sum2 = f2_add(sum2, v[c][e]);
        }
      }
    }
    prefetch(g + gridDim.x);
    float s;
    {
      float a0, a1;
      f2_unpack(sum2, a0, a1);
      s = a0 + a1;
    }
    // mean over the row: warp shuffle, then the row's WPR warps in fixed order
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0 && rloc < RPC) red[0][rloc][wr] = s;
    __syncthreads();
    float tot = 0.0f;
    if (rloc < RPC) {
#pragma unroll
      for (int i = 0; i < WPR; ++i) tot += red[0][rloc][i];
    }
    const float mean = tot * inv_h;
    const rln_f2 mean2 = f2_pack(mean, mean);
    rln_f2 sq2 = 0ull;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = ((c * WPR + wr) * 32 + lane) * 8;
      if (live && col < p.H) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[c][e] = f2_sub(v[c][e], mean2);  // centred from here on
          sq2 = f2_fma(v[c][e], v[c][e], sq2);
        }
      }
    }
    float s2;
    {
      float a0, a1;
      f2_unpack(sq2, a0, a1);
      s2 = a0 + a1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    if (lane == 0 && rloc < RPC) red[1][rloc][wr] = s2;
    __syncthreads();
    float tot2 = 0.0f;
    if (rloc < RPC) {
#pragma unroll
      for (int i = 0; i < WPR; ++i) tot2 += red[1][rloc][i];
    }
    const float rstd = 1.0f / sqrtf(tot2 * inv_h + p.eps);
    if (p.stats && live && wr == 0 && lane == 0)
      *reinterpret_cast<float2*>(p.stats + 2 * row) = make_float2(mean, rstd);
    const rln_f2 rstd2 = f2_pack(rstd, rstd);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = ((c * WPR + wr) * 32 + lane) * 8;
      if (live && col < p.H) {
        rln_f2 gm[4], bt[4];
        if (p.gamma) {
          const ulonglong2 ga = reinterpret_cast<const ulonglong2*>(p.gamma + col)[0];
          const ulonglong2 gb = reinterpret_cast<const ulonglong2*>(p.gamma + col)[1];
          gm[0] = ga.x; gm[1] = ga.y; gm[2] = gb.x; gm[3] = gb.y;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) gm[e] = f2_pack(1.0f, 1.0f);
        }
        if (p.beta) {
          const ulonglong2 ba = reinterpret_cast<const ulonglong2*>(p.beta + col)[0];
          const ulonglong2 bb = reinterpret_cast<const ulonglong2*>(p.beta + col)[1];
          bt[0] = ba.x; bt[1] = ba.y; bt[2] = bb.x; bt[3] = bb.y;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) bt[e] = 0ull;
        }
        float y[8];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          f2_unpack(f2_fma(v[c][e], f2_mul(rstd2, gm[e]), bt[e]), y[2 * e], y[2 * e + 1]);
        store8(p, base + col, y);
      }
    }
    __syncthreads();  // `red` is reused by the next row group
  }
}

// ------------------------------------------------ rows staged by bulk copies
// The same operation with each row's inputs (X and the f32 partials) brought
// into shared memory by untiled bulk copies (cp.async.bulk) instead of loaded
// by the threads: one thread issues a row's copies `nst` rows ahead of the
// row the CTA is reducing, so several rows per CTA are in flight from HBM
// while the CTA runs a row's two reductions, and the threads hold only their
// own 8-element chunks in registers.  One CTA of 256 threads walks rows
// blockIdx.x, blockIdx.x + gridDim.x, ...; thread i's chunk c covers columns
// (c * 256 + i) * 8 .. + 7.  The statistics are the two-pass ones of the
// register kernel (mean, then the variance of the centred values; warp
// shuffles, then the warps' sums in warp order), so results are repeatable.
// Stage layout: [X row][partial 0 row][partial 1 row]..., each a multiple of
// 16 bytes (H % 8 == 0).
namespace rlb {
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int MAX_STAGE_SMEM = 200 * 1024;  // stages x stage bytes of one CTA
}

__device__ __forceinline__ void rlb_issue_row(const ReduceLnArgs& p, long long row, uint8_t* dst, uint64_t* bar,
                                              uint32_t xbytes, uint32_t pbytes) {
  mbar_arrive_expect_tx(bar, xbytes + static_cast<uint32_t>(p.nparts) * pbytes);
  const uint8_t* xsrc = static_cast<const uint8_t*>(p.X) + row * xbytes;
  bulk_load_1d(dst, xsrc, xbytes, bar);
  for (int q = 0; q < p.nparts; ++q) {
    const float* src = p.parts ? p.parts + q * p.part_stride : p.part_ptr[q];
    bulk_load_1d(dst + xbytes + q * pbytes, src + row * p.H, pbytes, bar);
  }
}

template <int CH>
__global__ void __launch_bounds__(rlb::THREADS) reduce_residual_ln_bulk_kernel(const ReduceLnArgs p, int nst,
                                                                              int stage_bytes) {
  extern __shared__ __align__(128) uint8_t rlb_smem[];
  __shared__ uint64_t full[4];
  __shared__ float red[2][2][rlb::WARPS];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t xbytes = static_cast<uint32_t>(p.H) * (p.x_bf16 ? 2u : 4u);
  const uint32_t pbytes = static_cast<uint32_t>(p.H) * 4u;
  if (tid == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
  }
  __syncthreads();
  griddep_wait();  // the partial sums come from the preceding kernel
  griddep_launch_dependents();
  const int n_my = blockIdx.x < p.S ? (p.S - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1 : 0;
  int issued = 0;  // rows whose copies thread 0 has issued
  if (tid == 0) {
    for (; issued < nst && issued < n_my; ++issued)
      rlb_issue_row(p, blockIdx.x + static_cast<long long>(issued) * gridDim.x, rlb_smem + issued * stage_bytes,
                    &full[issued], xbytes, pbytes);
  }
  const float inv_h = 1.0f / static_cast<float>(p.H);
  int i = 0;
  for (; i < n_my; ++i) {
    const int s = i % nst;
    const long long row = blockIdx.x + static_cast<long long>(i) * gridDim.x;
    const uint8_t* st = rlb_smem + s * stage_bytes;
    // Every thread waits for the row's copies; all take the same exit.
    const bool ok = mbar_wait(&full[s], static_cast<uint32_t>((i / nst) & 1));
    if (!__syncthreads_and(ok)) break;
    float v[CH][8];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (c * rlb::THREADS + tid) * 8;
      if (col < p.H) {
        if (p.x_bf16) {
          load8_bf16(reinterpret_cast<const __nv_bfloat16*>(st) + col, v[c]);
        } else {
          const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(st) + col);
          const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(st) + col + 4);
          v[c][0] = a.x; v[c][1] = a.y; v[c][2] = a.z; v[c][3] = a.w;
          v[c][4] = b.x; v[c][5] = b.y; v[c][6] = b.z; v[c][7] = b.w;
        }
        for (int q = 0; q < p.nparts; ++q) {
          const float* pr = reinterpret_cast<const float*>(st + xbytes + q * pbytes) + col;
          const float4 a = *reinterpret_cast<const float4*>(pr);
          const float4 b = *reinterpret_cast<const float4*>(pr + 4);
          v[c][0] += a.x; v[c][1] += a.y; v[c][2] += a.z; v[c][3] += a.w;
          v[c][4] += b.x; v[c][5] += b.y; v[c][6] += b.z; v[c][7] += b.w;
        }
      }
    }
    if (!p.apply_ln) {
      __syncthreads();  // every thread has its values: the stage may be refilled
      if (tid == 0 && i + nst < n_my) {
        fence_proxy_async_smem();
        rlb_issue_row(p, row + static_cast<long long>(nst) * gridDim.x, rlb_smem + s * stage_bytes, &full[s], xbytes,
                      pbytes);
        ++issued;
      }
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int col = (c * rlb::THREADS + tid) * 8;
        if (col < p.H) store8(p, row * p.H + col, v[c]);
      }
      continue;
    }
    float sum = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      if ((c * rlb::THREADS + tid) * 8 < p.H) {
#pragma unroll
        for (int e = 0; e < 8; ++e) sum += v[c][e];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) red[i & 1][0][warp] = sum;
    __syncthreads();
    // Every thread has read the stage: refill it with the row nst rows ahead.
    if (tid == 0 && i + nst < n_my) {
      fence_proxy_async_smem();
      rlb_issue_row(p, row + static_cast<long long>(nst) * gridDim.x, rlb_smem + s * stage_bytes, &full[s], xbytes,
                    pbytes);
      ++issued;
    }
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < rlb::WARPS; ++w) tot += red[i & 1][0][w];
    const float mean = tot * inv_h;
    float s2 = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      if ((c * rlb::THREADS + tid) * 8 < p.H) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float d = v[c][e] - mean;
          s2 = fmaf(d, d, s2);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    if (lane == 0) red[i & 1][1][warp] = s2;
    __syncthreads();
    float tot2 = 0.0f;
#pragma unroll
    for (int w = 0; w < rlb::WARPS; ++w) tot2 += red[i & 1][1][w];
    const float rstd = 1.0f / sqrtf(tot2 * inv_h + p.eps);
    if (p.stats && tid == 0) *reinterpret_cast<float2*>(p.stats + 2 * row) = make_float2(mean, rstd);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (c * rlb::THREADS + tid) * 8;
      if (col < p.H) {
        float gm[8], bt[8];
        if (p.gamma) load8_f32_keep(p.gamma + col, gm);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) gm[e] = 1.0f;
        }
        if (p.beta) load8_f32_keep(p.beta + col, bt);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) bt[e] = 0.0f;
        }
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = fmaf((v[c][e] - mean) * rstd, gm[e], bt[e]);
        store8(p, row * p.H + col, y);
      }
    }
  }
  // After an error exit, rows issued but not consumed may still have copies in
  // flight: let them land (bounded) before the CTA's shared memory is released.
  if (tid == 0) {
    for (int j = i; j < issued; ++j) {
      const uint32_t a = smem_u32(&full[j % nst]);
      const long long t0 = clock64();
      while (!mbar_try_wait(a, static_cast<uint32_t>((j / nst) & 1)) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
    }
  }
}

}  // namespace tp
