// Per-head non-causal softmax attention on the 5th-generation tensor cores:
//
//   O_h = softmax(Q_h K_h^T / sqrt(d)) V_h       (d = 128, no mask)
//
// Heads are independent, which is what lets the QKV projection be split by
// head across tensor-parallel shards with no exchange until the O projection
// ("1. 张量并行：Tensor Parallelism" §1.2.2; "TP到底在切什么" §2.2 figure 4).
//
// One CTA per (head, 128 query rows), 6 warps:
//   warp 0      TMA: the Q tile once, then K_j and V_j tiles (128 keys each)
//               into a 2-stage ring.
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer.
//               S_j = Q K_j^T into one of two TMEM score buffers, then
//               O += P_{j-1} V_{j-1}, so the scores of block j are computed
//               while the softmax warps still work on block j-1.
//   warps 2..5  one query row per thread: row max, exp2, row sum (online
//               softmax), P_j as bf16 into shared memory in the 128-byte
//               swizzled K-major layout the MMA reads, rescaling of the O
//               accumulator in TMEM, final O / l to global memory.
// The running max is only raised when a block's max exceeds it by more than
// 2^8 (log2 domain), so O is rescaled rarely; P then stays below 2^8, which
// bf16 and the f32 accumulator carry without loss of relative precision.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm_tcgen05.cuh"
#include "ptx.cuh"

namespace tp {

namespace attn {
constexpr int D = 128;            // head dimension
constexpr int BQ = 128;           // query rows per CTA
constexpr int BKV = 128;          // keys per block
constexpr int NUM_THREADS = 192;
constexpr int HALF_BYTES = BQ * 64 * 2;   // one 64-column (128 B) box of 128 rows: 16 KiB
constexpr int TILE_BYTES = 2 * HALF_BYTES;  // 128 rows x 128 bf16: 32 KiB
constexpr int SMEM_BYTES = TILE_BYTES * (1 + 2 + 2 + 1) + 1024 + 256;
constexpr uint32_t IDESC_QK = idesc_bf16_f32(BQ, BKV, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BQ, D, false, true);
constexpr uint32_t TMEM_COLS = 512;       // S0 [0,128), S1 [128,256), O [256,384)
constexpr float RESCALE_THRESHOLD = 8.0f;
}  // namespace attn

struct AttnArgs {
  CUtensorMap tmQKV;   // [S, 3H] bf16, box {64, 128}
  void* O;             // [S, H] bf16, head h in columns h*D ..
  int S, H, nh;
  int heads_per_shard;
  int shard_cols;      // 3 * heads_per_shard * D: width of one shard's [Q|K|V] block
  float scale_log2;    // log2(e) / sqrt(D)
};

__global__ void __launch_bounds__(attn::NUM_THREADS, 1) attn_fwd_kernel(const __grid_constant__ AttnArgs a) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + TILE_BYTES;        // 2 stages
  uint8_t* sV = sK + 2 * TILE_BYTES;    // 2 stages
  uint8_t* sP = sV + 2 * TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + TILE_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* kv_empty = bars + 5;  // [2]
  uint64_t* s_full = bars + 7;    // [2]
  uint64_t* s_free = bars + 9;    // [2]
  uint64_t* p_full = bars + 11;
  uint64_t* pv_done = bars + 12;
  uint64_t* drain = bars + 13;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 14);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * BQ;
  const int h = blockIdx.y;
  const int shard = h / a.heads_per_shard;
  const int hj = h % a.heads_per_shard;
  const int Hs = a.heads_per_shard * D;
  const int qcol = shard * a.shard_cols + hj * D;
  const int kcol = qcol + Hs;
  const int vcol = qcol + 2 * Hs;
  const int nkv = a.S / BKV;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
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
  const uint32_t tS0 = tmem_base;
  const uint32_t tO = tmem_base + 256;

  if (warp == 0) {
    if (lane == 0) {
      int armed[5] = {-1, -1, -1, -1, -1};  // q, k0, k1, v0, v1
      bool ok = true;
      mbar_arrive_expect_tx(q_full, TILE_BYTES);
      armed[0] = 0;
      tma_load_2d(sQ, &a.tmQKV, qcol, q0, q_full);
      tma_load_2d(sQ + HALF_BYTES, &a.tmQKV, qcol + 64, q0, q_full);
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(&kv_empty[st], ph ^ 1)) { ok = false; break; }
        uint8_t* dk = sK + st * TILE_BYTES;
        uint8_t* dv = sV + st * TILE_BYTES;
        mbar_arrive_expect_tx(&k_full[st], TILE_BYTES);
        armed[1 + st] = static_cast<int>(ph);
        tma_load_2d(dk, &a.tmQKV, kcol, j * BKV, &k_full[st]);
        tma_load_2d(dk + HALF_BYTES, &a.tmQKV, kcol + 64, j * BKV, &k_full[st]);
        mbar_arrive_expect_tx(&v_full[st], TILE_BYTES);
        armed[3 + st] = static_cast<int>(ph);
        tma_load_2d(dv, &a.tmQKV, vcol, j * BKV, &v_full[st]);
        tma_load_2d(dv + HALF_BYTES, &a.tmQKV, vcol + 64, j * BKV, &v_full[st]);
      }
      if (!ok) {
        uint64_t* bl[5] = {q_full, &k_full[0], &k_full[1], &v_full[0], &v_full[1]};
        for (int i = 0; i < 5; ++i) {
          if (armed[i] < 0) continue;
          const uint32_t ad = smem_u32(bl[i]);
          const long long t0 = clock64();
          while (!mbar_try_wait(ad, static_cast<uint32_t>(armed[i])) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t p_addr = smem_u32(sP);
      for (int j = 0; j <= nkv && ok; ++j) {
        if (j < nkv) {
          const int b = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          if (!mbar_wait(&k_full[b], ph) || !mbar_wait(&s_free[b], ph ^ 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sK + b * TILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            umma_bf16(tS0 + b * 128, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024),
                      IDESC_QK, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[b]);
        }
        if (j >= 1) {
          const int i = j - 1;
          const int st = i & 1;
          const uint32_t ph = (i >> 1) & 1;
          if (!mbar_wait(&v_full[st], ph) || !mbar_wait(p_full, i & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sV + st * TILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk) {
            const uint32_t poff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            umma_bf16(tO, sdesc_sw128(p_addr + poff, 16, 1024), sdesc_sw128(v_addr + kk * 2048, HALF_BYTES, 1024),
                      IDESC_PV, (i > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(pv_done);
          umma_commit(&kv_empty[st]);
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
    const int q = warp & 3;
    const int r = q * 32 + lane;  // query row inside the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    float m_run = -INFINITY;
    float l_run = 0.0f;
    bool ok = true;
    uint8_t* prow0 = sP + r * 128;               // keys 0..63 of this row
    uint8_t* prow1 = sP + HALF_BYTES + r * 128;  // keys 64..127
    for (int j = 0; j < nkv; ++j) {
      const int b = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[b], (j >> 1) & 1))) { ok = false; break; }
      tc_fence_after();
      float s[BKV];
      {
        uint32_t u[32];
#pragma unroll
        for (int c = 0; c < BKV / 32; ++c) {
          tmem_ld_32x32b_x32(tS0 + b * 128 + lane_off + c * 32, u);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(u[e]);
        }
      }
      tc_fence_before();
      mbar_arrive(&s_free[b]);
      float mx = s[0];
#pragma unroll
      for (int e = 1; e < BKV; ++e) mx = fmaxf(mx, s[e]);
      const float m_blk = mx * a.scale_log2;
      const bool resc = m_blk > m_run + RESCALE_THRESHOLD;
      float alpha = 1.0f;
      if (resc) {
        alpha = exp2_fast(m_run - m_blk);  // 0 on the first block
        m_run = m_blk;
      }
      float sum = 0.0f;
      uint32_t pk[BKV / 2];
#pragma unroll
      for (int e = 0; e < BKV; e += 2) {
        const float p0 = exp2_fast(fmaf(s[e], a.scale_log2, -m_run));
        const float p1 = exp2_fast(fmaf(s[e + 1], a.scale_log2, -m_run));
        __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
        const float2 back = __bfloat1622float2(hp);
        sum += back.x + back.y;
        pk[e / 2] = *reinterpret_cast<uint32_t*>(&hp);
      }
      l_run = l_run * alpha + sum;
      if (j > 0) {
        // P_{j-1} V_{j-1} must be done before sP is overwritten and O rescaled.
        if (!__all_sync(0xffffffffu, mbar_wait(pv_done, (j - 1) & 1))) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            tmem_ld_32x32b_x32(tO + lane_off + c * 32, u);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
            tmem_st_32x32b_x32(tO + lane_off + c * 32, u);
          }
          tmem_wait_st();
        }
      }
      // P row -> shared memory, 128-byte swizzle: 16-byte chunk c of row r is
      // stored at chunk (c ^ (r & 7)).
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        uint8_t* rowp = c < 8 ? prow0 : prow1;
        const int cc = c & 7;
        uint4 w = make_uint4(pk[c * 4 + 0], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
        *reinterpret_cast<uint4*>(rowp + ((cc ^ (r & 7)) << 4)) = w;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(pv_done, (nkv - 1) & 1))) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      const int grow = q0 + r;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.O) + static_cast<long long>(grow) * a.H + h * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld_32x32b_x32(tO + lane_off + c * 32, u);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(u[g * 8 + 0]) * inv, __uint_as_float(u[g * 8 + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(u[g * 8 + 2]) * inv, __uint_as_float(u[g * 8 + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(u[g * 8 + 4]) * inv, __uint_as_float(u[g * 8 + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(u[g * 8 + 6]) * inv, __uint_as_float(u[g * 8 + 7]) * inv);
          *reinterpret_cast<uint4*>(orow + c * 32 + g * 8) = w;
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
