// Persistent, warp-specialised bf16 GEMM on the 5th-generation tensor cores.
//
//   C[M, :] = Act( A[M, K] * B[K, N] )          with B given as t shards.
//
// Two ways B is sharded, the two splits of the tensor-parallel linear layers:
//  * column mode — B = [B_0 | B_1 | ... ] split by columns ("按列切分",
//    "张量并行：千亿大模型突破单卡显存限制的底层技术" §2.1; "1. 张量并行：Tensor
//    Parallelism" §1.1 列切分).  Shard s writes its own column slice of C, so
//    the concatenation (the AllGather of the multi-GPU form) is a layout.
//  * row mode — B = [B_0; B_1; ...] split by rows, A's columns split to match
//    ("按行切分" §2.2; "外积和切分", eq. (1.1)).  The K loop walks the shards in
//    order and every shard's partial product accumulates into the same TMEM
//    accumulator, so the sum (the AllReduce of the multi-GPU form) costs no
//    extra memory traffic.
//
// Design (sm_100a): one CTA per SM, 6 warps.
//   warp 0      TMA producer: A box 128x64 (K-major, 128B swizzle), B as four
//               64(k) x 64(n) boxes (N-major, 128B swizzle), 4-stage ring.
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//               (M=128, N=256, K=16 per instruction, f32 accumulate in TMEM).
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, activation, store.
// The accumulator is double-buffered in TMEM (2 x 256 of the 512 columns), so
// the epilogue of tile i overlaps the main loop of tile i+1.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace tp {

constexpr int MAX_SHARDS = 8;

enum : int { ACT_NONE = 0, ACT_GELU_TANH = 1, ACT_GELU_ERF = 2, ACT_RELU = 3 };

namespace gemm {
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;          // 16 KiB
constexpr int B_BOX_N = 64;                   // 64 bf16 = one 128-byte swizzle row
constexpr int B_BOX_BYTES = BK * B_BOX_N * 2; // 8 KiB
constexpr int B_BOXES = BN / B_BOX_N;         // 4
constexpr int B_BYTES = BK * BN * 2;          // 32 KiB
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES) + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, /*a_mn=*/false, /*b_mn=*/true);
}  // namespace gemm

struct GemmArgs {
  CUtensorMap tmA;               // A [M, K] bf16 row-major, box {64, 128}
  CUtensorMap tmB[MAX_SHARDS];   // B shard s, bf16 row-major [rows, cols], box {64, 64}
  void* C;                       // output, row-major, ldc elements per row
  long long ldc;
  int M;
  int N;                         // column mode: t * shard_n; row mode: shard_n
  int t;
  int row_mode;
  int shard_n;                   // columns of each B shard
  int shard_k;                   // rows of each B shard
  int n_blocks_per_shard;        // column mode
  int k_blocks_per_shard;        // row mode (column mode: k blocks of K)
  int m_blocks, n_blocks, k_blocks;
  int act;
  int out_f32;
};

__device__ __forceinline__ float apply_act(float u, int act) {
  if (act == ACT_GELU_TANH) {
    const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
    return 0.5f * u * (1.0f + tanh_fast(k0 * fmaf(0.044715f * u, u * u, u)));
  } else if (act == ACT_GELU_ERF) {
    return 0.5f * u * (1.0f + erff(u * 0.7071067811865476f));
  } else if (act == ACT_RELU) {
    return fmaxf(u, 0.0f);
  }
  return u;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Tile coordinates shared by the three roles.
struct TileCoord {
  int m0;        // first row
  int shard;     // column mode: shard owning the tile's columns
  int n_in;      // first column inside the B operand (shard-local in column mode)
  int out_col0;  // first column of C
  int n_valid;   // valid columns in this tile (<= BN)
};

__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& p, int tile) {
  TileCoord c;
  const int mb = tile % p.m_blocks;
  const int nb = tile / p.m_blocks;
  c.m0 = mb * gemm::BM;
  if (!p.row_mode) {
    c.shard = nb / p.n_blocks_per_shard;
    c.n_in = (nb % p.n_blocks_per_shard) * gemm::BN;
    c.out_col0 = c.shard * p.shard_n + c.n_in;
    c.n_valid = min(gemm::BN, p.shard_n - c.n_in);
  } else {
    c.shard = 0;
    c.n_in = nb * gemm::BN;
    c.out_col0 = c.n_in;
    c.n_valid = min(gemm::BN, p.shard_n - c.n_in);
  }
  return c;
}

__global__ void __launch_bounds__(gemm::NUM_THREADS, 1) gemm_tcgen05_kernel(const __grid_constant__ GemmArgs p) {
  using namespace gemm;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    for (int s = 0; s < p.t; ++s) tma_prefetch_desc(&p.tmB[s]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int num_tiles = p.m_blocks * p.n_blocks;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int armed[STAGES];  // parity of the last phase this thread armed per stage
#pragma unroll
      for (int s = 0; s < STAGES; ++s) armed[s] = -1;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const TileCoord tc = tile_coord(p, tile);
        const int nboxes = min(B_BOXES, (tc.n_valid + B_BOX_N - 1) / B_BOX_N);
        const uint32_t bytes = A_BYTES + nboxes * B_BOX_BYTES;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          int shard, a_x, b_y;
          if (p.row_mode) {
            shard = kb / p.k_blocks_per_shard;
            b_y = (kb % p.k_blocks_per_shard) * BK;
            a_x = shard * p.shard_k + b_y;
          } else {
            shard = tc.shard;
            b_y = kb * BK;
            a_x = b_y;
          }
          mbar_arrive_expect_tx(&full[stage], bytes);
          armed[stage] = static_cast<int>(phase);
          tma_load_2d(sA + stage * A_BYTES, &p.tmA, a_x, tc.m0, &full[stage]);
          for (int j = 0; j < nboxes; ++j)
            tma_load_2d(sB + stage * B_BYTES + j * B_BOX_BYTES, &p.tmB[shard], tc.n_in + j * B_BOX_N, b_y,
                        &full[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // Let every copy already issued land before the CTA can exit.
        for (int s = 0; s < STAGES; ++s) {
          if (armed[s] < 0) continue;
          const uint32_t a = smem_u32(&full[s]);
          const long long t0 = clock64();
          while (!mbar_try_wait(a, static_cast<uint32_t>(armed[s])) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // A: K-major, 16 k-elements = 32 bytes further along the swizzled row.
            const uint64_t ad = sdesc_sw128(a0 + kk * 32, 16, 1024);
            // B: N-major, 16 k-rows = 2 x (8 rows x 128 B) further; 64-column
            // chunks are B_BOX_BYTES apart (leading offset), 8-row groups 1 KiB.
            const uint64_t bd = sdesc_sw128(b0 + kk * 2048, B_BOX_BYTES, 1024);
            umma_bf16(d_tmem, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      if (!ok) {
        // Wait (bounded) for every MMA already issued before TMEM is freed.
        umma_commit(drain);
        const uint32_t a = smem_u32(drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(a, 0) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_local = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const TileCoord tc = tile_coord(p, tile);
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase))) break;
      tc_fence_after();
      const int grow = tc.m0 + row_local;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      for (int c = 0; c < BN / 32; ++c) {
        if (c * 32 >= tc.n_valid) break;  // uniform across the CTA
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + c * 32, r);
        tmem_wait_ld();
        if (grow < p.M) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int col = c * 32 + g * 8;
            if (col < tc.n_valid) {
              float v[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) v[e] = apply_act(__uint_as_float(r[g * 8 + e]), p.act);
              const long long off = static_cast<long long>(grow) * p.ldc + tc.out_col0 + col;
              if (p.out_f32) {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.C) + off);
                dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                dst[1] = make_float4(v[4], v[5], v[6], v[7]);
              } else {
                uint4 w;
                w.x = pack_bf16x2(v[0], v[1]);
                w.y = pack_bf16x2(v[2], v[3]);
                w.z = pack_bf16x2(v[4], v[5]);
                w.w = pack_bf16x2(v[6], v[7]);
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + off) = w;
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
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
