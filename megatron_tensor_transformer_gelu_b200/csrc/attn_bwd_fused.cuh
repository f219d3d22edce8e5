// The softmax attention's backward per head, with P and dS kept on chip:
//
//   S = Q K^T,  P = 2^(S scale_log2 - lse2),  dP = dO V^T,
//   dS = P (dP - D) / sqrt d        (D = rowsum(dO * O), lse2 from the forward)
//   dV = P^T dO,  dK = dS^T Q,  dQ = dS K
//
// Two kernels, each a loop over one head's tiles with every product on the
// 5th-generation tensor cores and the elementwise steps in between on 128
// threads, one TMEM lane (one row) each:
//
//   attn_bwd_dkv_kernel  one CTA per (128 keys, head): K_j and V_j stay in
//     shared memory while 64-query tiles Q_i, dO_i (and their lse2 and D
//     values) stream through a 3-stage ring.  Per query tile:
//       S^T = K_j Q_i^T and dP^T = V_j dO_i^T into TMEM (lane = key);
//       P^T and dS^T, as bf16 pairs over the first 32 columns of each;
//       dV_j += P^T dO_i and dK_j += dS^T Q_i with A read from TMEM.
//   attn_bwd_dq_kernel   one CTA per (128 queries, head): Q_i and dO_i stay,
//     128-key tiles K_j, V_j stream through a 2-stage ring.  Per key tile:
//       S = Q_i K_j^T and dP = dO_i V_j^T (lane = query);
//       dS as bf16 pairs over the first 64 columns of dP;
//       dQ_i += dS K_j with A read from TMEM.
//
// S, P, dP and dS never reach memory, and no result is reduced across CTAs:
// the key-major kernel sums dV and dK over the queries in TMEM, the
// query-major kernel sums dQ over the keys.  The price is computing S and dP
// twice.  In the key-major kernel the S^T and dP^T of a query tile are 64
// columns wide, so TMEM holds two of each (4 x 64 f32 columns) besides the
// 128-column dV and dK: the tensor core computes tile t + 2's S^T and dP^T
// (and tile t's last products) while the elementwise threads work on tile
// t + 1.  The query-major kernel keeps 128-key tiles and one S and dP (with
// 64-key tiles and two buffers it measured slower).  Roles: warp 0 loads (TMA),
// warp 1 allocates TMEM and issues the MMAs from one thread, warps 2..5 run
// the elementwise steps and the epilogue.  A buffer of S and dP is reused
// by a later tile whose S and dP are issued after the products that read the
// buffer's P and dS, by the same thread, so they overwrite them only once
// those have completed.  Every wait is bounded.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm_tcgen05.cuh"
#include "ptx.cuh"

namespace tp {

namespace attb {
constexpr int D = 128;                       // head dimension
constexpr int BT = 128;                      // rows of the resident tile (keys or queries): TMEM lanes
constexpr int BS = 64;                       // rows of a streamed tile: columns of S and dP
// Elementwise warpgroups per kernel: each takes its own columns of every tile.
// Measured (ncu, one box): the query-major kernel 282 us with two against
// 291-293 us with one, the key-major kernel 366-369 us with one against 376
// us with two.
#ifndef TP_ATTB_DKV_EWG
#define TP_ATTB_DKV_EWG 1
#endif
#ifndef TP_ATTB_DQ_EWG
#define TP_ATTB_DQ_EWG 2
#endif
constexpr int DKV_EWG = TP_ATTB_DKV_EWG;
constexpr int DQ_EWG = TP_ATTB_DQ_EWG;
// warp 0 loads, warp 1 MMAs, the rest elementwise
constexpr int DKV_THREADS = 64 + 128 * DKV_EWG;
constexpr int DQ_THREADS = 64 + 128 * DQ_EWG;
constexpr int STAGES = 3;                    // streamed tiles in flight
constexpr int HALF_T = BT * 64 * 2;          // one 64-column (128 B) box of a resident tile: 16 KiB
constexpr int HALF_S = BS * 64 * 2;          // the same for a streamed tile: 8 KiB
constexpr int TILE_T = 2 * HALF_T;           // 32 KiB
constexpr int TILE_S = 2 * HALF_S;           // 16 KiB
constexpr int VEC_BYTES = BS * 4;            // one streamed tile's lse2 or D values
constexpr int SMEM_DKV = 2 * TILE_T + STAGES * (2 * TILE_S + 2 * VEC_BYTES) + 1024 + 256;
constexpr int DQ_STAGES = 2;                 // key tiles (128 rows) in flight in the query-major kernel
constexpr int SMEM_DQ = 2 * TILE_T + DQ_STAGES * 2 * TILE_T + 1024 + 256;
constexpr uint32_t IDESC_SS = idesc_bf16_f32(BT, BS, false, false);  // S^T, dP^T: A, B K-major (smem)
constexpr uint32_t IDESC_SQ = idesc_bf16_f32(BT, BT, false, false);  // S, dP of the query-major kernel
constexpr uint32_t IDESC_TB = idesc_bf16_f32(BT, D, false, true);    // A from TMEM, B MN-major
constexpr uint32_t TMEM_COLS = 512;
}  // namespace attb

struct AttnBwdArgs {
  CUtensorMap tmQKV_t;      // [S, 3H] bf16, box {64, 128}: resident tiles
  CUtensorMap tmQKV_s;      // [S, 3H] bf16, box {64, 64}: streamed tiles
  CUtensorMap tmdO_t;       // [S, nh D] bf16, box {64, 128}
  CUtensorMap tmdO_s;       // [S, nh D] bf16, box {64, 64}
  const float* lse2;        // [nh, S]
  const float* Dvec;        // [nh, S]
  __nv_bfloat16* dQKV;      // [S, 3H], laid out as QKV
  long long ld_qkv;         // 3H
  int S, nh;
  int heads_per_shard;
  int shard_cols;           // 3 * heads_per_shard * D
  float scale_log2;         // log2(e) / sqrt(D)
  float scale;              // 1 / sqrt(D)
};

// K-major (smem) operand of a tile whose two 64-column boxes are `half`
// bytes apart, for the kk-th 16-element K step; MN-major B operand of such a
// tile for the kk-th 16-row K step.
__device__ __forceinline__ uint64_t attb_kmajor(uint32_t tile, int half, int kk) {
  return sdesc_sw128(tile + (kk >> 2) * half + (kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t attb_mnmajor(uint32_t tile, int half, int kk) {
  return sdesc_sw128(tile + kk * 2048, static_cast<uint32_t>(half), 1024);
}

// f32 accumulator columns [c0 * 32, c1 * 32) of row r (TMEM lane = r) as bf16
// into dst (which points at column 0).
__device__ __forceinline__ void attb_store_row(uint32_t t_row, __nv_bfloat16* dst, int c0 = 0,
                                               int c1 = attb::D / 32) {
  for (int c = c0; c < c1; ++c) {
    uint32_t u[32];
    tmem_ld_32x32b_x32(t_row + c * 32, u);
    tmem_wait_ld();
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint4 w;
      w.x = pack_bf16x2(__uint_as_float(u[g * 8 + 0]), __uint_as_float(u[g * 8 + 1]));
      w.y = pack_bf16x2(__uint_as_float(u[g * 8 + 2]), __uint_as_float(u[g * 8 + 3]));
      w.z = pack_bf16x2(__uint_as_float(u[g * 8 + 4]), __uint_as_float(u[g * 8 + 5]));
      w.w = pack_bf16x2(__uint_as_float(u[g * 8 + 6]), __uint_as_float(u[g * 8 + 7]));
      *reinterpret_cast<uint4*>(dst + c * 32 + g * 8) = w;
    }
  }
}

// P, dS as bf16 pairs: of `ewg` elementwise warpgroups, group g owns columns
// [g n, (g + 1) n) of a buffer (n = cols / ewg) and stores the pairs of its
// rows' values there, from its first column on (only over columns it has
// read).  The packed column that holds rows [16 kk, 16 kk + 16) of the K
// dimension:
__device__ __forceinline__ uint32_t attb_packed_col(int kk, int cols, int ewg) {
  const int n = cols / ewg, q = 16 * kk, g = q / n;
  return static_cast<uint32_t>(g * n + (q - g * n) / 2);
}

// Wait (bounded) for the copies a producer thread armed before it gave up.
__device__ __forceinline__ void attb_drain(uint64_t* const* bars, const int* armed, int n) {
  for (int i = 0; i < n; ++i) {
    if (armed[i] < 0) continue;
    const uint32_t ad = smem_u32(bars[i]);
    const long long t0 = clock64();
    while (!mbar_try_wait(ad, static_cast<uint32_t>(armed[i])) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
  }
}

// The MMA thread's wait for an in-flight drain after a failed wait.
__device__ __forceinline__ void attb_mma_drain(uint64_t* drain) {
  umma_commit(drain);
  const uint32_t ad = smem_u32(drain);
  const long long t0 = clock64();
  while (!mbar_try_wait(ad, 0) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
}

__global__ void __launch_bounds__(attb::DKV_THREADS, 1) attn_bwd_dkv_kernel(const __grid_constant__ AttnBwdArgs a) {
  using namespace attb;
  constexpr int EWG = DKV_EWG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + TILE_T;
  uint8_t* sQ = sV + TILE_T;                     // STAGES tiles
  uint8_t* sdO = sQ + STAGES * TILE_S;           // STAGES tiles
  float* sL = reinterpret_cast<float*>(sdO + STAGES * TILE_S);  // STAGES x BS lse2 values
  float* sD = sL + STAGES * BS;                                  // STAGES x BS D values
  uint64_t* bars = reinterpret_cast<uint64_t*>(sD + STAGES * BS);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;                   // [STAGES]
  uint64_t* q_empty = q_full + STAGES;           // [STAGES]
  uint64_t* s_full = q_empty + STAGES;           // [2]: S and dP of a buffer computed
  uint64_t* p_full = s_full + 2;                 // [2]: P and dS of a buffer written
  uint64_t* acc_full = p_full + 2;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int j0 = blockIdx.x * BT;                // this CTA's keys [j0, j0 + BT)
  const int h = blockIdx.y;
  const int Hs = a.heads_per_shard * D;
  const int qcol = (h / a.heads_per_shard) * a.shard_cols + (h % a.heads_per_shard) * D;
  const int kcol = qcol + Hs, vcol = qcol + 2 * Hs, ocol = h * D;
  const int nq = a.S / BS;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128 * EWG);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&a.tmQKV_t);
    tma_prefetch_desc(&a.tmQKV_s);
    tma_prefetch_desc(&a.tmdO_s);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // S buffers at columns [0, 64) and [64, 128), dP buffers at [128, 192) and [192, 256)
  const uint32_t tS = tmem_base, tdP = tmem_base + 128, tdV = tmem_base + 256, tdK = tmem_base + 384;
  griddep_wait();  // QKV, dO, lse2 and D come from preceding kernels
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int armed[1 + STAGES];
      uint64_t* armed_bar[1 + STAGES] = {kv_full};
      for (int i = 0; i < STAGES; ++i) armed_bar[1 + i] = &q_full[i];
      for (int i = 0; i <= STAGES; ++i) armed[i] = -1;
      mbar_arrive_expect_tx(kv_full, 2 * TILE_T);
      armed[0] = 0;
      tma_load_2d(sK, &a.tmQKV_t, kcol, j0, kv_full);
      tma_load_2d(sK + HALF_T, &a.tmQKV_t, kcol + 64, j0, kv_full);
      tma_load_2d(sV, &a.tmQKV_t, vcol, j0, kv_full);
      tma_load_2d(sV + HALF_T, &a.tmQKV_t, vcol + 64, j0, kv_full);
      bool ok = true;
      for (int i = 0; i < nq; ++i) {
        const int st = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&q_empty[st], ph ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&q_full[st], 2 * TILE_S + 2 * VEC_BYTES);
        armed[1 + st] = static_cast<int>(ph);
        uint8_t* q = sQ + st * TILE_S;
        uint8_t* o = sdO + st * TILE_S;
        tma_load_2d(q, &a.tmQKV_s, qcol, i * BS, &q_full[st]);
        tma_load_2d(q + HALF_S, &a.tmQKV_s, qcol + 64, i * BS, &q_full[st]);
        tma_load_2d(o, &a.tmdO_s, ocol, i * BS, &q_full[st]);
        tma_load_2d(o + HALF_S, &a.tmdO_s, ocol + 64, i * BS, &q_full[st]);
        const long long v0 = static_cast<long long>(h) * a.S + static_cast<long long>(i) * BS;
        bulk_load_1d(sL + st * BS, a.lse2 + v0, VEC_BYTES, &q_full[st]);
        bulk_load_1d(sD + st * BS, a.Dvec + v0, VEC_BYTES, &q_full[st]);
      }
      if (!ok) attb_drain(armed_bar, armed, 1 + STAGES);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(kv_full, 0);
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      // S^T = K_j Q_i^T and dP^T = V_j dO_i^T of query tile i into buffer i & 1.
      auto issue_sdp = [&](int i) -> bool {
        const int st = i % STAGES, b = i & 1;
        if (!mbar_wait(&q_full[st], (i / STAGES) & 1)) return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQ + st * TILE_S), o_addr = smem_u32(sdO + st * TILE_S);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tS + b * BS, attb_kmajor(k_addr, HALF_T, kk), attb_kmajor(q_addr, HALF_S, kk), IDESC_SS,
                    kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tdP + b * BS, attb_kmajor(v_addr, HALF_T, kk), attb_kmajor(o_addr, HALF_S, kk), IDESC_SS,
                    kk > 0 ? 1u : 0u);
        umma_commit(&s_full[b]);
        return true;
      };
      for (int i = 0; i < 2 && i < nq && ok; ++i) ok = issue_sdp(i);
      for (int i = 0; i < nq && ok; ++i) {
        const int st = i % STAGES, b = i & 1;
        // P^T over buffer b of S^T, dS^T over buffer b of dP^T (K = the tile's queries).
        if (!mbar_wait(&p_full[b], (i >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQ + st * TILE_S), o_addr = smem_u32(sdO + st * TILE_S);
#pragma unroll
        for (int kk = 0; kk < BS / 16; ++kk)
          umma_bf16_tmem_a(tdV, tS + b * BS + attb_packed_col(kk, BS, EWG), attb_mnmajor(o_addr, HALF_S, kk), IDESC_TB,
                           (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < BS / 16; ++kk)
          umma_bf16_tmem_a(tdK, tdP + b * BS + attb_packed_col(kk, BS, EWG), attb_mnmajor(q_addr, HALF_S, kk), IDESC_TB,
                           (i > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&q_empty[st]);
        // Tile i + 2 reuses buffer b: issued after the products above.
        if (i + 2 < nq && !issue_sdp(i + 2)) { ok = false; break; }
      }
      if (ok) umma_commit(acc_full);
      else attb_mma_drain(drain);
    }
  } else {
    // ------------------------------------------ elementwise and epilogue
    const int r = (warp & 3) * 32 + lane;                 // key row of the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int g = (warp - 2) >> 2;                        // elementwise warpgroup
    constexpr int GC = BS / EWG;                          // its columns (queries) of a tile
    bool ok = true;
    for (int i = 0; i < nq; ++i) {
      const int st = i % STAGES, b = i & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[b], (i >> 1) & 1))) { ok = false; break; }
      // lse2 and D of this query tile arrived with Q_i.
      if (!__all_sync(0xffffffffu, mbar_wait(&q_full[st], (i / STAGES) & 1))) { ok = false; break; }
      tc_fence_after();
      const float* L = sL + st * BS;
      const float* Dv = sD + st * BS;
      const uint32_t tSb = tS + b * BS + lane_off + g * GC, tdPb = tdP + b * BS + lane_off + g * GC;
#pragma unroll
      for (int c = 0; c < GC / 32; ++c) {
        uint32_t us[32], ud[32], pp[16], pd[16];
        tmem_ld_32x32b_x32(tSb + c * 32, us);
        tmem_ld_32x32b_x32(tdPb + c * 32, ud);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int q = g * GC + c * 32 + 2 * e;
          const float p0 = exp2_fast(fmaf(__uint_as_float(us[2 * e]), a.scale_log2, -L[q]));
          const float p1 = exp2_fast(fmaf(__uint_as_float(us[2 * e + 1]), a.scale_log2, -L[q + 1]));
          const float d0 = (p0 * (__uint_as_float(ud[2 * e]) - Dv[q])) * a.scale;
          const float d1 = (p1 * (__uint_as_float(ud[2 * e + 1]) - Dv[q + 1])) * a.scale;
          pp[e] = pack_bf16x2(p0, p1);
          pd[e] = pack_bf16x2(d0, d1);
        }
        // The group's columns [16c, 16c + 16) hold its queries [32c, 32c + 32)
        // as pairs; they lie within the columns it has already read.
        tmem_st_32x32b_x16(tSb + c * 16, pp);
        tmem_st_32x32b_x16(tdPb + c * 16, pd);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(acc_full, 0))) {
      tc_fence_after();
      __nv_bfloat16* row = a.dQKV + static_cast<long long>(j0 + r) * a.ld_qkv;
      if (EWG == 1 || g == 0) attb_store_row(tdV + lane_off, row + vcol);
      if (EWG == 1 || g == 1) attb_store_row(tdK + lane_off, row + kcol);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

__global__ void __launch_bounds__(attb::DQ_THREADS, 1) attn_bwd_dq_kernel(const __grid_constant__ AttnBwdArgs a) {
  using namespace attb;
  constexpr int EWG = DQ_EWG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + TILE_T;
  uint8_t* sK = sdO + TILE_T;                    // DQ_STAGES tiles
  uint8_t* sV = sK + DQ_STAGES * TILE_T;         // DQ_STAGES tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + DQ_STAGES * TILE_T);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;                  // [DQ_STAGES]
  uint64_t* kv_empty = kv_full + DQ_STAGES;      // [DQ_STAGES]
  uint64_t* s_full = kv_empty + DQ_STAGES;
  uint64_t* p_full = s_full + 1;
  uint64_t* acc_full = p_full + 1;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int i0 = blockIdx.x * BT;                // this CTA's queries [i0, i0 + BT)
  const int h = blockIdx.y;
  const int Hs = a.heads_per_shard * D;
  const int qcol = (h / a.heads_per_shard) * a.shard_cols + (h % a.heads_per_shard) * D;
  const int kcol = qcol + Hs, vcol = qcol + 2 * Hs, ocol = h * D;
  const int nk = a.S / BT;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < DQ_STAGES; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128 * EWG);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&a.tmQKV_t);
    tma_prefetch_desc(&a.tmdO_t);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t tS = tmem_base, tdP = tmem_base + 128, tdQ = tmem_base + 256;
  griddep_wait();  // QKV, dO, lse2 and D come from preceding kernels
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int armed[1 + DQ_STAGES];
      uint64_t* armed_bar[1 + DQ_STAGES] = {q_full};
      for (int i = 0; i < DQ_STAGES; ++i) armed_bar[1 + i] = &kv_full[i];
      for (int i = 0; i <= DQ_STAGES; ++i) armed[i] = -1;
      mbar_arrive_expect_tx(q_full, 2 * TILE_T);
      armed[0] = 0;
      tma_load_2d(sQ, &a.tmQKV_t, qcol, i0, q_full);
      tma_load_2d(sQ + HALF_T, &a.tmQKV_t, qcol + 64, i0, q_full);
      tma_load_2d(sdO, &a.tmdO_t, ocol, i0, q_full);
      tma_load_2d(sdO + HALF_T, &a.tmdO_t, ocol + 64, i0, q_full);
      bool ok = true;
      for (int j = 0; j < nk; ++j) {
        const int st = j % DQ_STAGES;
        const uint32_t ph = (j / DQ_STAGES) & 1;
        if (!mbar_wait(&kv_empty[st], ph ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&kv_full[st], 2 * TILE_T);
        armed[1 + st] = static_cast<int>(ph);
        uint8_t* k = sK + st * TILE_T;
        uint8_t* v = sV + st * TILE_T;
        tma_load_2d(k, &a.tmQKV_t, kcol, j * BT, &kv_full[st]);
        tma_load_2d(k + HALF_T, &a.tmQKV_t, kcol + 64, j * BT, &kv_full[st]);
        tma_load_2d(v, &a.tmQKV_t, vcol, j * BT, &kv_full[st]);
        tma_load_2d(v + HALF_T, &a.tmQKV_t, vcol + 64, j * BT, &kv_full[st]);
      }
      if (!ok) attb_drain(armed_bar, armed, 1 + DQ_STAGES);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0);
      const uint32_t q_addr = smem_u32(sQ), o_addr = smem_u32(sdO);
      for (int j = 0; j < nk && ok; ++j) {
        const int st = j % DQ_STAGES;
        if (!mbar_wait(&kv_full[st], (j / DQ_STAGES) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * TILE_T), v_addr = smem_u32(sV + st * TILE_T);
        // S = Q_i K_j^T, dP = dO_i V_j^T (K = d).
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tS, attb_kmajor(q_addr, HALF_T, kk), attb_kmajor(k_addr, HALF_T, kk), IDESC_SQ,
                    kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tdP, attb_kmajor(o_addr, HALF_T, kk), attb_kmajor(v_addr, HALF_T, kk), IDESC_SQ,
                    kk > 0 ? 1u : 0u);
        umma_commit(s_full);
        // dS over dP's first 64 columns (K = keys).
        if (!mbar_wait(p_full, j & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk)
          umma_bf16_tmem_a(tdQ, tdP + attb_packed_col(kk, BT, EWG), attb_mnmajor(k_addr, HALF_T, kk), IDESC_TB,
                           (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&kv_empty[st]);
      }
      if (ok) umma_commit(acc_full);
      else attb_mma_drain(drain);
    }
  } else {
    // ------------------------------------------ elementwise and epilogue
    const int r = (warp & 3) * 32 + lane;                 // query row of the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int g = (warp - 2) >> 2;                        // elementwise warpgroup
    constexpr int GC = BT / EWG;                          // its columns (keys) of a tile
    const long long v0 = static_cast<long long>(h) * a.S + i0 + r;
    const float lse = a.lse2[v0], Dr = a.Dvec[v0];
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, j & 1))) { ok = false; break; }
      tc_fence_after();
      const uint32_t tSg = tS + lane_off + g * GC, tdPg = tdP + lane_off + g * GC;
#pragma unroll
      for (int c = 0; c < GC / 32; ++c) {
        uint32_t us[32], ud[32], pd[16];
        tmem_ld_32x32b_x32(tSg + c * 32, us);
        tmem_ld_32x32b_x32(tdPg + c * 32, ud);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = exp2_fast(fmaf(__uint_as_float(us[2 * e]), a.scale_log2, -lse));
          const float p1 = exp2_fast(fmaf(__uint_as_float(us[2 * e + 1]), a.scale_log2, -lse));
          pd[e] = pack_bf16x2((p0 * (__uint_as_float(ud[2 * e]) - Dr)) * a.scale,
                              (p1 * (__uint_as_float(ud[2 * e + 1]) - Dr)) * a.scale);
        }
        // The group's columns [16c, 16c + 16) hold its keys [32c, 32c + 32)
        // as pairs; they lie within the columns it has already read.
        tmem_st_32x32b_x16(tdPg + c * 16, pd);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(acc_full, 0))) {
      tc_fence_after();
      attb_store_row(tdQ + lane_off, a.dQKV + static_cast<long long>(i0 + r) * a.ld_qkv + qcol,
                     g * (D / 32 / EWG), (g + 1) * (D / 32 / EWG));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace tp
