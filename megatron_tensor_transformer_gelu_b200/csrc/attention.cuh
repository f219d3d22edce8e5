// Per-head non-causal softmax attention on the 5th-generation tensor cores:
//
//   O_h = softmax(Q_h K_h^T / sqrt(d)) V_h       (d = 128, no mask)
//
// Heads are independent, which is what lets the QKV projection be split by
// head across tensor-parallel shards with no exchange until the O projection
// ("1. 张量并行：Tensor Parallelism" §1.2.2; "TP到底在切什么" §2.2 figure 4).
//
// One CTA per (head, 256 query rows) = two 128-row query tiles that share
// every K and V tile, 11 warps:
//   warp 0      TMA: Q0, Q1 once, then K_j (128 keys) into a 2-stage ring.
//   warp 10     TMA: V_j into a 2-stage ring.
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer, in the
//               order P0_j V_j, S0_{j+1}, P1_j V_j, S1_{j+1} (S_t = Q_t K^T).
//   warps 2..5  softmax of tile 0, one query row per thread;
//   warps 6..9  softmax of tile 1.  While one group runs its exponentials
//               (bound by the MUFU units), the other loads scores, reduces,
//               or waits for its MMAs, so the two tiles ping-pong.
// TMEM: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512) f32 columns.
// P_t (bf16 pairs) is written over the first 64 columns of S_t once S_t has
// been read and P_t(j-1) V has been consumed, and is fed to the P V product
// straight from TMEM (no shared-memory round trip); S_t(j+1) is issued after
// P_t(j) V_j by the same thread.
// The running max is only raised when a block's max exceeds it by more than
// 2^8 (log2 domain), so O is rescaled in TMEM rarely; P then stays below
// 2^8, which bf16 and the f32 accumulator carry without loss of relative
// precision.
//
// Last-wave key split.  The (head, 256-row) units are equal, so a grid of U
// units on P resident CTAs ends with a partial wave of U mod P units.  Those
// last units may be run as two CTAs each, over key blocks [0, kv_half) and
// [kv_half, nkv): the same softmax-weighted sums over fewer keys.  Per warp
// (32 query rows of a tile) the two halves meet through a flag pair in global
// memory: each takes the claim flag with an atomic exchange of the launch's
// epoch; the first to take it stores its unnormalised O rows and its (m, l)
// and publishes the ready flag; the second waits (bounded) for ready, and
// merges
//     m = max(m1, m2),  l = l1 2^(m1-m) + l2 2^(m2-m),
//     O = (O1 2^(m1-m) + O2 2^(m2-m)) / l
// (the online softmax's combination of two key ranges), then stores O and
// the row's log2 denominator.  The merge is symmetric in the two halves, so
// results do not depend on which half arrives first.  No CTA ever waits for
// a CTA that has not finished its main loop, so no wait can deadlock.  The
// flags carry the launch's epoch, so flags left by an earlier launch that
// gave up never match; the merging half clears the pair after use, so the
// replays of a captured launch (one epoch for all of them) start unclaimed.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm_tcgen05.cuh"
#include "ptx.cuh"

namespace tp {

namespace attn {
constexpr int D = 128;            // head dimension
constexpr int BQ = 128;           // query rows per tile
constexpr int TILES = 2;          // query tiles per CTA
constexpr int BKV = 128;          // keys per block
constexpr int NUM_THREADS = 352;  // 11 warps
#ifndef TP_ATTN_K_STAGES
#define TP_ATTN_K_STAGES 2
#endif
#ifndef TP_ATTN_V_STAGES
#define TP_ATTN_V_STAGES 2
#endif
constexpr int K_STAGES = TP_ATTN_K_STAGES;
constexpr int V_STAGES = TP_ATTN_V_STAGES;
constexpr int HALF_BYTES = BQ * 64 * 2;     // one 64-column (128 B) box of 128 rows: 16 KiB
constexpr int TILE_BYTES = 2 * HALF_BYTES;  // 128 rows x 128 bf16: 32 KiB
constexpr int SMEM_BYTES = TILE_BYTES * (TILES + K_STAGES + V_STAGES) + 1024 + 256;
constexpr uint32_t IDESC_QK = idesc_bf16_f32(BQ, BKV, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BQ, D, false, true);
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;
#ifndef TP_ATTN_EXP2_POLY_EVERY
#define TP_ATTN_EXP2_POLY_EVERY 0
#endif
// Softmax arithmetic on f32 pairs (f32x2 scale and row sum, three-input max).
#ifndef TP_ATTN_X2
#define TP_ATTN_X2 1
#endif
constexpr int EXP2_POLY_EVERY = TP_ATTN_EXP2_POLY_EVERY;  // 0: every exponential on the MUFU unit
constexpr int EXP2_POLY_MOD = EXP2_POLY_EVERY > 0 ? EXP2_POLY_EVERY : 1;
}  // namespace attn

struct AttnArgs {
  CUtensorMap tmQKV;   // [S, 3H] bf16, box {64, 128}
  void* O;             // [S, H] bf16, head h in columns h*D ..
  int S, H, nh;
  int heads_per_shard;
  int shard_cols;      // 3 * heads_per_shard * D: width of one shard's [Q|K|V] block
  float scale_log2;    // log2(e) / sqrt(D)
  float* lse2;         // optional [nh, S]: log2 of each row's softmax denominator, in the
                       // units of the scores times scale_log2 (what a backward pass
                       // needs to rebuild P = 2^(s scale_log2 - lse2))
  // Units (head, 256 query rows) in launch order: unit u = head u / nq, query
  // block u % nq.  Blocks [0, whole) run units 0..whole-1 over every key;
  // blocks whole + 2i and whole + 2i + 1 run unit whole + i over key blocks
  // [0, kv_half) and [kv_half, nkv).
  int nq;
  int whole;
  int kv_half;
  float* part_o;                   // split scratch: [split units][2][4][32 col groups][32 rows] float4
  float* part_ml;                  // [split units][2][4][2][32]: m and l of the stored rows
  unsigned long long* part_flags;  // [split units][2][4][2]: claim, ready
  unsigned long long epoch;        // this launch's flag value
};

// Atomic exchange with acquire-release semantics at GPU scope.
__device__ __forceinline__ unsigned long long flag_exchange(unsigned long long* addr, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.exch.b64 %0, [%1], %2;" : "=l"(old) : "l"(addr), "l"(v) : "memory");
  return old;
}

__global__ void __launch_bounds__(attn::NUM_THREADS, 1) attn_fwd_kernel(const __grid_constant__ AttnArgs a) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                            // TILES tiles
  uint8_t* sK = sQ + TILES * TILE_BYTES;         // K_STAGES stages
  uint8_t* sV = sK + K_STAGES * TILE_BYTES;      // V_STAGES stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + V_STAGES * TILE_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;                   // [K_STAGES]
  uint64_t* k_empty = k_full + K_STAGES;         // [K_STAGES]
  uint64_t* v_full = k_empty + K_STAGES;         // [V_STAGES]
  uint64_t* v_empty = v_full + V_STAGES;         // [V_STAGES]
  uint64_t* s_full = v_empty + V_STAGES;         // [TILES]
  uint64_t* p_full = s_full + TILES;             // [TILES]
  uint64_t* pv_done = p_full + TILES;            // [TILES]
  uint64_t* drain = pv_done + TILES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nkv = a.S / BKV;
  int unit = blockIdx.x, kb0 = 0, nkb = nkv, su = -1;  // su: split unit index, -1 when whole
  if (unit >= a.whole) {
    const int v = unit - a.whole;
    su = v >> 1;
    unit = a.whole + su;
    kb0 = (v & 1) ? a.kv_half : 0;
    nkb = (v & 1) ? nkv - a.kv_half : a.kv_half;
  }
  const int q0 = (unit % a.nq) * (TILES * BQ);
  const int h = unit / a.nq;
  const int shard = h / a.heads_per_shard;
  const int hj = h % a.heads_per_shard;
  const int Hs = a.heads_per_shard * D;
  const int qcol = shard * a.shard_cols + hj * D;
  const int kcol = qcol + Hs;
  const int vcol = qcol + 2 * Hs;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < K_STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < V_STAGES; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int t = 0; t < TILES; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&pv_done[t], 1);
    }
    mbar_init(drain, 1);
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&a.tmQKV);
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  griddep_wait();  // Q, K and V come from the preceding kernel
  griddep_launch_dependents();

  if (warp == 0 || warp == 10) {
    // ---------------------------------------------- producers (Q + K, V)
    if (lane == 0) {
      const bool is_k = warp == 0;
      const int nst = is_k ? K_STAGES : V_STAGES;
      uint64_t* fullb = is_k ? k_full : v_full;
      uint64_t* emptyb = is_k ? k_empty : v_empty;
      uint8_t* base = is_k ? sK : sV;
      const int col = is_k ? kcol : vcol;
      // armed[st]: the phase stage st's barrier expects (-1: none); armed[QS]: the Q load's
      constexpr int QS = K_STAGES > V_STAGES ? K_STAGES : V_STAGES;
      int armed[QS + 1];
#pragma unroll
      for (int i = 0; i <= QS; ++i) armed[i] = -1;
      bool ok = true;
      if (is_k) {
        // Tiles past S (an odd tile count) are zero-filled by the TMA.
        mbar_arrive_expect_tx(q_full, TILES * TILE_BYTES);
        armed[QS] = 0;
        for (int t = 0; t < TILES; ++t) {
          tma_load_2d(sQ + t * TILE_BYTES, &a.tmQKV, qcol, q0 + t * BQ, q_full);
          tma_load_2d(sQ + t * TILE_BYTES + HALF_BYTES, &a.tmQKV, qcol + 64, q0 + t * BQ, q_full);
        }
      }
      for (int j = 0; j < nkb; ++j) {
        const int st = j % nst;
        const uint32_t ph = (j / nst) & 1;
        if (!mbar_wait(&emptyb[st], ph ^ 1)) { ok = false; break; }
        uint8_t* d = base + st * TILE_BYTES;
        mbar_arrive_expect_tx(&fullb[st], TILE_BYTES);
        armed[st] = static_cast<int>(ph);
        tma_load_2d(d, &a.tmQKV, col, (kb0 + j) * BKV, &fullb[st]);
        tma_load_2d(d + HALF_BYTES, &a.tmQKV, col + 64, (kb0 + j) * BKV, &fullb[st]);
      }
      if (!ok) {
        for (int i = 0; i <= QS; ++i) {
          if (armed[i] < 0 || (i < QS && i >= nst)) continue;
          const uint32_t ad = smem_u32(i == QS ? q_full : &fullb[i]);
          const long long t0 = clock64();
          while (!mbar_try_wait(ad, static_cast<uint32_t>(armed[i])) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0);
      const uint32_t q_addr = smem_u32(sQ);
      // S_t(j) = Q_t K_j^T into columns [t*128, t*128+128).  Tile 0 waits for
      // K_j; tile 1 releases its stage.
      auto issue_s = [&](int j, int t) -> bool {
        const int ks = j % K_STAGES;
        if (t == 0) {
          if (!mbar_wait(&k_full[ks], (j / K_STAGES) & 1)) return false;
          tc_fence_after();
        }
        const uint32_t k_addr = smem_u32(sK + ks * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          umma_bf16(tmem_base + t * 128, sdesc_sw128(q_addr + t * TILE_BYTES + off, 16, 1024),
                    sdesc_sw128(k_addr + off, 16, 1024), IDESC_QK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[t]);
        if (t == TILES - 1) umma_commit(&k_empty[ks]);
        return true;
      };
      for (int t = 0; t < TILES && ok && nkb > 0; ++t) ok = issue_s(0, t);
      // Per block: P0 V, S0(j+1), P1 V, S1(j+1).  Tile 0's next scores are
      // ready while tile 1 is still in its exponentials, and the reverse.
      for (int j = 0; j < nkb && ok; ++j) {
        const int vs = j % V_STAGES;
        if (!mbar_wait(&v_full[vs], (j / V_STAGES) & 1)) { ok = false; break; }
        const uint32_t v_addr = smem_u32(sV + vs * TILE_BYTES);
        for (int t = 0; t < TILES && ok; ++t) {
          // P_t(j) sits in the first 64 columns of S_t once the softmax arrived.
          if (!mbar_wait(&p_full[t], j & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t tP = tmem_base + t * 128;
          const uint32_t tO = tmem_base + 256 + t * 128;
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk)
            umma_bf16_tmem_a(tO, tP + kk * 8, sdesc_sw128(v_addr + kk * 2048, HALF_BYTES, 1024), IDESC_PV,
                             (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&pv_done[t]);
          if (t == TILES - 1) umma_commit(&v_empty[vs]);
          // S_t(j+1) overwrites P_t(j): issued after P_t(j) V_j above.
          if (j + 1 < nkb && !issue_s(j + 1, t)) { ok = false; break; }
        }
      }
      if (!ok) {
        umma_commit(drain);
        const uint32_t ad = smem_u32(drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(ad, 0) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
      }
    }
  } else {
    // --------------------------------------------------- softmax / epilogue
    const int tile = warp < 6 ? 0 : 1;                 // warps 2..5 -> tile 0, 6..9 -> tile 1
    const int q = warp & 3;                            // TMEM lane quarter
    const int r = q * 32 + lane;                       // query row inside the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t tS = tmem_base + tile * 128 + lane_off;
    const uint32_t tO = tmem_base + 256 + tile * 128 + lane_off;
    float m_run = -INFINITY;
    float l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkb; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[tile], j & 1))) { ok = false; break; }
      tc_fence_after();
      float s[BKV];
      {
        uint32_t u0[32], u1[32], u2[32], u3[32];
        tmem_ld_32x32b_x32(tS + 0, u0);
        tmem_ld_32x32b_x32(tS + 32, u1);
        tmem_ld_32x32b_x32(tS + 64, u2);
        tmem_ld_32x32b_x32(tS + 96, u3);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          s[e] = __uint_as_float(u0[e]);
          s[32 + e] = __uint_as_float(u1[e]);
          s[64 + e] = __uint_as_float(u2[e]);
          s[96 + e] = __uint_as_float(u3[e]);
        }
      }
      // Row max with 8 independent chains (three-input max), then a tree.
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = s[i];
#if TP_ATTN_X2
#pragma unroll
      for (int e = 8; e + 16 <= BKV; e += 16)
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = max3f(m8[i], s[e + i], s[e + 8 + i]);
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = fmaxf(m8[i], s[BKV - 8 + i]);
      const float mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
#else
#pragma unroll
      for (int e = 8; e < BKV; e += 8)
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmaxf(m8[i], s[e + i]);
      const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
#endif
      const float m_blk = mx * a.scale_log2;
      const bool resc = m_blk > m_run + RESCALE_THRESHOLD;
      float alpha = 1.0f;
      if (resc) {
        alpha = exp2_fast(m_run - m_blk);  // 0 on the first block
        m_run = m_blk;
      }
      // p = 2^(s * scale_log2 - m) in f32, kept as bf16 pairs for the P V
      // product; the row sum adds the f32 values in independent chains.
      // One pair in EXP2_POLY_EVERY is evaluated on the FMA pipe instead of
      // the MUFU unit, whose exponentials bound this loop.
      uint32_t pk0[32], pk1[32];
#if TP_ATTN_X2
      // Scaling and the row sum on pairs of lanes (f32x2): half the FMA-pipe
      // instructions.
      const unsigned long long sc2 = f2_pack(a.scale_log2, a.scale_log2);
      const unsigned long long nm2 = f2_pack(-m_run, -m_run);
      unsigned long long sum4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int e = 0; e < BKV; e += 2) {
        const bool poly = EXP2_POLY_EVERY > 0 && (e / 2) % EXP2_POLY_MOD == EXP2_POLY_MOD - 1;
        float x0, x1, p0, p1;
        f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), sc2, nm2), x0, x1);
        if (poly) {
          exp2_poly3_pair(x0, x1, p0, p1);
        } else {
          p0 = exp2_fast(x0);
          p1 = exp2_fast(x1);
        }
        sum4[(e / 2) & 3] = f2_add(sum4[(e / 2) & 3], f2_pack(p0, p1));
        if (e < 64) pk0[e / 2] = pack_bf16x2(p0, p1);
        else pk1[(e - 64) / 2] = pack_bf16x2(p0, p1);
      }
      float sum;
      {
        float a0, a1;
        f2_unpack(f2_add(f2_add(sum4[0], sum4[1]), f2_add(sum4[2], sum4[3])), a0, a1);
        sum = a0 + a1;
      }
#else
      float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < BKV; e += 2) {
        const bool poly = EXP2_POLY_EVERY > 0 && (e / 2) % EXP2_POLY_MOD == EXP2_POLY_MOD - 1;
        const float x0 = fmaf(s[e], a.scale_log2, -m_run);
        const float x1 = fmaf(s[e + 1], a.scale_log2, -m_run);
        const float p0 = poly ? exp2_poly(x0) : exp2_fast(x0);
        const float p1 = poly ? exp2_poly(x1) : exp2_fast(x1);
        sum8[(e / 2) & 7] += p0 + p1;
        if (e < 64) pk0[e / 2] = pack_bf16x2(p0, p1);
        else pk1[(e - 64) / 2] = pack_bf16x2(p0, p1);
      }
      const float sum = ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
#endif
      l_run = l_run * alpha + sum;
      if (j > 0) {
        // P_t(j-1) V_{j-1} must be done before P_t(j) replaces it and O_t is
        // rescaled.
        if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[tile], (j - 1) & 1))) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            tmem_ld_32x32b_x32(tO + c * 32, u);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
            tmem_st_32x32b_x32(tO + c * 32, u);
          }
        }
      }
      // P_t(j): 128 keys of row r as 64 columns of bf16 pairs over S_t.
      tmem_st_32x32b_x32(tS + 0, pk0);
      tmem_st_32x32b_x32(tS + 32, pk1);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[tile]);
    }
    const bool tile_valid = q0 + tile * BQ < a.S;  // the second tile of an odd tile count is not stored
    if (ok && __all_sync(0xffffffffu, mbar_wait(&pv_done[tile], (nkb - 1) & 1)) && tile_valid) {
      tc_fence_after();
      // Split unit: the first half to claim this warp's rows stores them and
      // is done; the second merges them with its own.
      bool merge = false;
      float4* po = nullptr;
      float* pml = nullptr;
      if (su >= 0) {
        const int slot = (su * TILES + tile) * 4 + q;
        unsigned long long* flags = a.part_flags + 2 * slot;
        po = reinterpret_cast<float4*>(a.part_o) + static_cast<long long>(slot) * (D / 4) * 32;
        pml = a.part_ml + slot * 64;
        unsigned long long prev = 0;
        if (lane == 0) prev = flag_exchange(&flags[0], a.epoch);
        merge = __shfl_sync(0xffffffffu, prev == a.epoch ? 1 : 0, 0) != 0;
        if (!merge) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            tmem_ld_32x32b_x32(tO + c * 32, u);
            tmem_wait_ld();
#pragma unroll
            for (int g = 0; g < 8; ++g)
              __stcg(po + (c * 8 + g) * 32 + lane,
                     make_float4(__uint_as_float(u[g * 4 + 0]), __uint_as_float(u[g * 4 + 1]),
                                 __uint_as_float(u[g * 4 + 2]), __uint_as_float(u[g * 4 + 3])));
          }
          __stcg(pml + lane, m_run);
          __stcg(pml + 32 + lane, l_run);
          __threadfence();
          __syncwarp();
          if (lane == 0) flag_publish(&flags[1], a.epoch);
        } else {
          bool ready = true;
          if (lane == 0) ready = flag_wait_eq(&flags[1], a.epoch);
          ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
          __threadfence();
          if (!ready) merge = false;
          // Both halves are done with the flag pair: clear it, so a replay of
          // this launch (a CUDA graph keeps its epoch) finds it unclaimed.
          if (ready && lane == 0) {
            flag_publish(&flags[0], 0ull);
            flag_publish(&flags[1], 0ull);
          }
        }
        if (!merge) po = nullptr;  // stored (or gave up): nothing to write here
      }
      if (su < 0 || po) {
        // Row scale: 1 / l, or for a merge 2^(m_own - m) / l and 2^(m_other - m) / l,
        // formed the same way whichever half is "own", so the sum is symmetric.
        float s_own = 1.0f, s_oth = 0.0f, m_fin = m_run, l_fin = l_run;
        if (po) {
          const float m_oth = __ldcg(pml + lane);
          const float l_oth = __ldcg(pml + 32 + lane);
          m_fin = fmaxf(m_run, m_oth);
          const float e_own = exp2_fast(m_run - m_fin), e_oth = exp2_fast(m_oth - m_fin);
          l_fin = __fadd_rn(__fmul_rn(l_run, e_own), __fmul_rn(l_oth, e_oth));
          const float inv = 1.0f / l_fin;
          s_own = __fmul_rn(e_own, inv);
          s_oth = __fmul_rn(e_oth, inv);
        } else {
          s_own = 1.0f / l_run;
        }
        const int grow = q0 + tile * BQ + r;
        if (a.lse2) a.lse2[static_cast<long long>(h) * a.S + grow] = m_fin + __log2f(l_fin);
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.O) + static_cast<long long>(grow) * a.H + h * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t u[32];
          tmem_ld_32x32b_x32(tO + c * 32, u);
          tmem_wait_ld();
          float o[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(u[e]) * s_own;
          if (po) {
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              const float4 v = __ldcg(po + (c * 8 + g) * 32 + lane);
              o[g * 4 + 0] = __fadd_rn(o[g * 4 + 0], __fmul_rn(v.x, s_oth));
              o[g * 4 + 1] = __fadd_rn(o[g * 4 + 1], __fmul_rn(v.y, s_oth));
              o[g * 4 + 2] = __fadd_rn(o[g * 4 + 2], __fmul_rn(v.z, s_oth));
              o[g * 4 + 3] = __fadd_rn(o[g * 4 + 3], __fmul_rn(v.w, s_oth));
            }
          }
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint4 w;
            w.x = pack_bf16x2(o[g * 8 + 0], o[g * 8 + 1]);
            w.y = pack_bf16x2(o[g * 8 + 2], o[g * 8 + 3]);
            w.z = pack_bf16x2(o[g * 8 + 4], o[g * 8 + 5]);
            w.w = pack_bf16x2(o[g * 8 + 6], o[g * 8 + 7]);
            *reinterpret_cast<uint4*>(orow + c * 32 + g * 8) = w;
          }
        }
      }
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
