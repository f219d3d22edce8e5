// The softmax attention's backward per head, with P and dS kept on chip:
//
//   S = Q K^T,  P = 2^(S scale_log2 - lse2),  dP = dO V^T,
//   dS = P (dP - D) / sqrt d        (D = rowsum(dO * O), lse2 from the forward)
//   dV = P^T dO,  dK = dS^T Q,  dQ = dS K
//
// Two kernels, each a loop over one head's 128-row tiles with every product
// on the 5th-generation tensor cores and the elementwise steps in between on
// 128 threads, one TMEM lane (one row) each:
//
//   attn_bwd_dkv_kernel  one CTA per (128 keys, head): K_j and V_j stay in
//     shared memory while the query tiles Q_i, dO_i (and their lse2 and D
//     values) stream through a 2-stage ring.  Per query tile:
//       S^T = K_j Q_i^T and dP^T = V_j dO_i^T into TMEM (lane = key);
//       P^T and dS^T, as bf16 pairs over the first 64 columns of each;
//       dV_j += P^T dO_i and dK_j += dS^T Q_i with A read from TMEM.
//   attn_bwd_dq_kernel   one CTA per (128 queries, head): Q_i and dO_i stay,
//     the key tiles K_j, V_j stream.  Per key tile:
//       S = Q_i K_j^T and dP = dO_i V_j^T (lane = query);
//       dS as bf16 pairs over the first 64 columns of dP;
//       dQ_i += dS K_j with A read from TMEM.
//
// S, P, dP and dS never reach memory, and no result is reduced across CTAs:
// the key-major kernel sums dV and dK over the queries in TMEM, the
// query-major kernel sums dQ over the keys.  The price is computing S and dP
// twice.  TMEM: 4 x 128 f32 columns (S, dP, dV, dK) and 3 x 128 (S, dP, dQ).
// Roles: warp 0 loads (TMA), warp 1 allocates TMEM and issues the MMAs from
// one thread, warps 2..5 run the elementwise steps and the epilogue.  The
// next tile's S and dP are issued after the current tile's last products by
// the same thread, so they overwrite P and dS only after those products have
// read them.  Every wait is bounded.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm_tcgen05.cuh"
#include "ptx.cuh"

namespace tp {

namespace attb {
constexpr int D = 128;                       // head dimension
constexpr int BT = 128;                      // rows of a key or query tile
constexpr int NUM_THREADS = 192;             // 6 warps
constexpr int STAGES = 2;
constexpr int HALF_BYTES = BT * 64 * 2;      // one 64-column (128 B) box of 128 rows: 16 KiB
constexpr int TILE_BYTES = 2 * HALF_BYTES;   // 128 rows x 128 bf16: 32 KiB
constexpr int VEC_BYTES = BT * 4;            // one tile's lse2 or D values
constexpr int SMEM_DKV = 2 * TILE_BYTES + STAGES * (2 * TILE_BYTES + 2 * VEC_BYTES) + 1024 + 256;
constexpr int SMEM_DQ = 2 * TILE_BYTES + STAGES * 2 * TILE_BYTES + 1024 + 256;
constexpr uint32_t IDESC_SS = idesc_bf16_f32(BT, BT, false, false);  // A, B K-major (smem)
constexpr uint32_t IDESC_TB = idesc_bf16_f32(BT, D, false, true);    // A from TMEM, B MN-major
constexpr uint32_t TMEM_COLS = 512;
}  // namespace attb

struct AttnBwdArgs {
  CUtensorMap tmQKV;        // [S, 3H] bf16, box {64, 128}
  CUtensorMap tmdO;         // [S, nh D] bf16, box {64, 128}
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

// The K-major (smem) operand of a 128 x 128 tile for the kk-th 16-element K
// step, and the MN-major B operand for the kk-th 16-row K step (the two
// 64-column halves HALF_BYTES apart).
__device__ __forceinline__ uint64_t attb_kmajor(uint32_t tile, int kk) {
  return sdesc_sw128(tile + (kk >> 2) * attb::HALF_BYTES + (kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t attb_mnmajor(uint32_t tile, int kk) {
  return sdesc_sw128(tile + kk * 2048, attb::HALF_BYTES, 1024);
}

// Row r's 128 f32 accumulator columns (TMEM lane = r) as bf16 into dst.
__device__ __forceinline__ void attb_store_row(uint32_t t_row, __nv_bfloat16* dst) {
#pragma unroll
  for (int c = 0; c < attb::D / 32; ++c) {
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

// Wait (bounded) for the copies a producer thread armed before it gave up.
__device__ __forceinline__ void attb_drain(uint64_t* const* bars, const int* armed, int n) {
  for (int i = 0; i < n; ++i) {
    if (armed[i] < 0) continue;
    const uint32_t ad = smem_u32(bars[i]);
    const long long t0 = clock64();
    while (!mbar_try_wait(ad, static_cast<uint32_t>(armed[i])) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
  }
}

__global__ void __launch_bounds__(attb::NUM_THREADS, 1) attn_bwd_dkv_kernel(const __grid_constant__ AttnBwdArgs a) {
  using namespace attb;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + TILE_BYTES;
  uint8_t* sQ = sV + TILE_BYTES;                 // STAGES tiles
  uint8_t* sdO = sQ + STAGES * TILE_BYTES;       // STAGES tiles
  float* sL = reinterpret_cast<float*>(sdO + STAGES * TILE_BYTES);  // STAGES x BT lse2 values
  float* sD = sL + STAGES * BT;                                      // STAGES x BT D values
  uint64_t* bars = reinterpret_cast<uint64_t*>(sD + STAGES * BT);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;                   // [STAGES]
  uint64_t* q_empty = q_full + STAGES;           // [STAGES]
  uint64_t* s_full = q_empty + STAGES;
  uint64_t* p_full = s_full + 1;
  uint64_t* acc_full = p_full + 1;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int j0 = blockIdx.x * BT;                // this CTA's keys [j0, j0 + BT)
  const int h = blockIdx.y;
  const int Hs = a.heads_per_shard * D;
  const int qcol = (h / a.heads_per_shard) * a.shard_cols + (h % a.heads_per_shard) * D;
  const int kcol = qcol + Hs, vcol = qcol + 2 * Hs, ocol = h * D;
  const int nq = a.S / BT;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&a.tmQKV);
    tma_prefetch_desc(&a.tmdO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
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
      mbar_arrive_expect_tx(kv_full, 2 * TILE_BYTES);
      armed[0] = 0;
      tma_load_2d(sK, &a.tmQKV, kcol, j0, kv_full);
      tma_load_2d(sK + HALF_BYTES, &a.tmQKV, kcol + 64, j0, kv_full);
      tma_load_2d(sV, &a.tmQKV, vcol, j0, kv_full);
      tma_load_2d(sV + HALF_BYTES, &a.tmQKV, vcol + 64, j0, kv_full);
      bool ok = true;
      for (int i = 0; i < nq; ++i) {
        const int st = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&q_empty[st], ph ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&q_full[st], 2 * TILE_BYTES + 2 * VEC_BYTES);
        armed[1 + st] = static_cast<int>(ph);
        uint8_t* q = sQ + st * TILE_BYTES;
        uint8_t* o = sdO + st * TILE_BYTES;
        tma_load_2d(q, &a.tmQKV, qcol, i * BT, &q_full[st]);
        tma_load_2d(q + HALF_BYTES, &a.tmQKV, qcol + 64, i * BT, &q_full[st]);
        tma_load_2d(o, &a.tmdO, ocol, i * BT, &q_full[st]);
        tma_load_2d(o + HALF_BYTES, &a.tmdO, ocol + 64, i * BT, &q_full[st]);
        const long long v0 = static_cast<long long>(h) * a.S + static_cast<long long>(i) * BT;
        bulk_load_1d(sL + st * BT, a.lse2 + v0, VEC_BYTES, &q_full[st]);
        bulk_load_1d(sD + st * BT, a.Dvec + v0, VEC_BYTES, &q_full[st]);
      }
      if (!ok) attb_drain(armed_bar, armed, 1 + STAGES);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(kv_full, 0);
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      for (int i = 0; i < nq && ok; ++i) {
        const int st = i % STAGES;
        if (!mbar_wait(&q_full[st], (i / STAGES) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQ + st * TILE_BYTES), o_addr = smem_u32(sdO + st * TILE_BYTES);
        // S^T = K_j Q_i^T, dP^T = V_j dO_i^T (K = d).
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tS, attb_kmajor(k_addr, kk), attb_kmajor(q_addr, kk), IDESC_SS, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tdP, attb_kmajor(v_addr, kk), attb_kmajor(o_addr, kk), IDESC_SS, kk > 0 ? 1u : 0u);
        umma_commit(s_full);
        // P^T over S^T's first 64 columns, dS^T over dP^T's (K = queries).
        if (!mbar_wait(p_full, i & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk)
          umma_bf16_tmem_a(tdV, tS + kk * 8, attb_mnmajor(o_addr, kk), IDESC_TB, (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk)
          umma_bf16_tmem_a(tdK, tdP + kk * 8, attb_mnmajor(q_addr, kk), IDESC_TB, (i > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&q_empty[st]);
      }
      if (ok) {
        umma_commit(acc_full);
      } else {
        umma_commit(drain);
        const uint32_t ad = smem_u32(drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(ad, 0) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
      }
    }
  } else {
    // ------------------------------------------ elementwise and epilogue
    const int r = (warp & 3) * 32 + lane;                 // key row of the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool ok = true;
    for (int i = 0; i < nq; ++i) {
      const int st = i % STAGES;
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, i & 1))) { ok = false; break; }
      // lse2 and D of this query tile arrived with Q_i.
      if (!__all_sync(0xffffffffu, mbar_wait(&q_full[st], (i / STAGES) & 1))) { ok = false; break; }
      tc_fence_after();
      const float* L = sL + st * BT;
      const float* Dv = sD + st * BT;
#pragma unroll
      for (int c = 0; c < BT / 32; ++c) {
        uint32_t us[32], ud[32], pp[16], pd[16];
        tmem_ld_32x32b_x32(tS + lane_off + c * 32, us);
        tmem_ld_32x32b_x32(tdP + lane_off + c * 32, ud);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int q = c * 32 + 2 * e;
          const float p0 = exp2_fast(fmaf(__uint_as_float(us[2 * e]), a.scale_log2, -L[q]));
          const float p1 = exp2_fast(fmaf(__uint_as_float(us[2 * e + 1]), a.scale_log2, -L[q + 1]));
          const float d0 = (p0 * (__uint_as_float(ud[2 * e]) - Dv[q])) * a.scale;
          const float d1 = (p1 * (__uint_as_float(ud[2 * e + 1]) - Dv[q + 1])) * a.scale;
          pp[e] = pack_bf16x2(p0, p1);
          pd[e] = pack_bf16x2(d0, d1);
        }
        // Columns [16c, 16c + 16) hold queries [32c, 32c + 32) as pairs; they
        // lie within the columns already read.
        tmem_st_32x32b_x16(tS + lane_off + c * 16, pp);
        tmem_st_32x32b_x16(tdP + lane_off + c * 16, pd);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(acc_full, 0))) {
      tc_fence_after();
      __nv_bfloat16* row = a.dQKV + static_cast<long long>(j0 + r) * a.ld_qkv;
      attb_store_row(tdV + lane_off, row + vcol);
      attb_store_row(tdK + lane_off, row + kcol);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

__global__ void __launch_bounds__(attb::NUM_THREADS, 1) attn_bwd_dq_kernel(const __grid_constant__ AttnBwdArgs a) {
  using namespace attb;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + TILE_BYTES;
  uint8_t* sK = sdO + TILE_BYTES;                // STAGES tiles
  uint8_t* sV = sK + STAGES * TILE_BYTES;        // STAGES tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + STAGES * TILE_BYTES);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;                  // [STAGES]
  uint64_t* kv_empty = kv_full + STAGES;         // [STAGES]
  uint64_t* s_full = kv_empty + STAGES;
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
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&a.tmQKV);
    tma_prefetch_desc(&a.tmdO);
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
      int armed[1 + STAGES];
      uint64_t* armed_bar[1 + STAGES] = {q_full};
      for (int i = 0; i < STAGES; ++i) armed_bar[1 + i] = &kv_full[i];
      for (int i = 0; i <= STAGES; ++i) armed[i] = -1;
      mbar_arrive_expect_tx(q_full, 2 * TILE_BYTES);
      armed[0] = 0;
      tma_load_2d(sQ, &a.tmQKV, qcol, i0, q_full);
      tma_load_2d(sQ + HALF_BYTES, &a.tmQKV, qcol + 64, i0, q_full);
      tma_load_2d(sdO, &a.tmdO, ocol, i0, q_full);
      tma_load_2d(sdO + HALF_BYTES, &a.tmdO, ocol + 64, i0, q_full);
      bool ok = true;
      for (int j = 0; j < nk; ++j) {
        const int st = j % STAGES;
        const uint32_t ph = (j / STAGES) & 1;
        if (!mbar_wait(&kv_empty[st], ph ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&kv_full[st], 2 * TILE_BYTES);
        armed[1 + st] = static_cast<int>(ph);
        uint8_t* k = sK + st * TILE_BYTES;
        uint8_t* v = sV + st * TILE_BYTES;
        tma_load_2d(k, &a.tmQKV, kcol, j * BT, &kv_full[st]);
        tma_load_2d(k + HALF_BYTES, &a.tmQKV, kcol + 64, j * BT, &kv_full[st]);
        tma_load_2d(v, &a.tmQKV, vcol, j * BT, &kv_full[st]);
        tma_load_2d(v + HALF_BYTES, &a.tmQKV, vcol + 64, j * BT, &kv_full[st]);
      }
      if (!ok) attb_drain(armed_bar, armed, 1 + STAGES);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0);
      const uint32_t q_addr = smem_u32(sQ), o_addr = smem_u32(sdO);
      for (int j = 0; j < nk && ok; ++j) {
        const int st = j % STAGES;
        if (!mbar_wait(&kv_full[st], (j / STAGES) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * TILE_BYTES), v_addr = smem_u32(sV + st * TILE_BYTES);
        // S = Q_i K_j^T, dP = dO_i V_j^T (K = d).
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tS, attb_kmajor(q_addr, kk), attb_kmajor(k_addr, kk), IDESC_SS, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tdP, attb_kmajor(o_addr, kk), attb_kmajor(v_addr, kk), IDESC_SS, kk > 0 ? 1u : 0u);
        umma_commit(s_full);
        // dS over dP's first 64 columns (K = keys).
        if (!mbar_wait(p_full, j & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk)
          umma_bf16_tmem_a(tdQ, tdP + kk * 8, attb_mnmajor(k_addr, kk), IDESC_TB, (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&kv_empty[st]);
      }
      if (ok) {
        umma_commit(acc_full);
      } else {
        umma_commit(drain);
        const uint32_t ad = smem_u32(drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(ad, 0) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
      }
    }
  } else {
    // ------------------------------------------ elementwise and epilogue
    const int r = (warp & 3) * 32 + lane;                 // query row of the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const long long v0 = static_cast<long long>(h) * a.S + i0 + r;
    const float lse = a.lse2[v0], Dr = a.Dvec[v0];
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, j & 1))) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < BT / 32; ++c) {
        uint32_t us[32], ud[32], pd[16];
        tmem_ld_32x32b_x32(tS + lane_off + c * 32, us);
        tmem_ld_32x32b_x32(tdP + lane_off + c * 32, ud);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = exp2_fast(fmaf(__uint_as_float(us[2 * e]), a.scale_log2, -lse));
          const float p1 = exp2_fast(fmaf(__uint_as_float(us[2 * e + 1]), a.scale_log2, -lse));
          pd[e] = pack_bf16x2((p0 * (__uint_as_float(ud[2 * e]) - Dr)) * a.scale,
                              (p1 * (__uint_as_float(ud[2 * e + 1]) - Dr)) * a.scale);
        }
        tmem_st_32x32b_x16(tdP + lane_off + c * 16, pd);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(acc_full, 0))) {
      tc_fence_after();
      attb_store_row(tdQ + lane_off, a.dQKV + static_cast<long long>(i0 + r) * a.ld_qkv + qcol);
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
