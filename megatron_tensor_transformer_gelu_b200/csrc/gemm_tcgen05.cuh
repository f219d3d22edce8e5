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
// Design (sm_100a), one CTA per SM, 6 warps, CG = 1 (one CTA per tile) or
// CG = 2 (a cluster of two CTAs on two SMs shares one tile through
// tcgen05.mma.cta_group::2):
//   warp 0      TMA producer.  Per stage each CTA loads its 128 rows of A
//               (box 128 x 64, K-major, 128-byte swizzle) and its BN/CG
//               columns of B (64 x 64 boxes, N-major, 128-byte swizzle).  In a
//               pair both CTAs' copies complete on the leader's barrier.
//   warp 1      TMEM allocator; lane 0 of the leader issues tcgen05.mma
//               (M = 128*CG, N = 256, K = 16 per instruction) into an f32
//               accumulator in TMEM and commits stage/accumulator releases
//               to both CTAs.
//   warps 2..5  epilogue: tcgen05.ld of this CTA's 128 accumulator rows,
//               activation (or another epilogue mode, see GemmArgs), a
//               swizzled staging write, and a TMA store per 128-byte chunk.
// The accumulator is double-buffered in TMEM (2 x 256 of the 512 columns), so
// the epilogue of tile i overlaps the main loop of tile i+1.  No load uses
// cluster multicast: every CTA fetches its own operand boxes.
//
// Wide tiles (WIDE = true, pairs only): a tile is 256 rows by up to 512
// columns, computed as two MMAs per K step (N = 256 into TMEM columns
// [0, 256), N = n2 into [256, 256 + n2)).  The accumulator then fills TMEM and
// is single-buffered, but every operand byte feeds more MACs and the tile
// count can be matched to the number of SM pairs (fewer, fuller waves).
//
// Narrow tiles (tile_n == 128, N-major B, not wide): one MMA of N = 128 per K
// step, each CTA of a pair holding 64 B columns, for shards of at most 128
// columns (no MMA work on columns past the shard).
//
// Column mode can give each shard its own A (a_per_shard): t independent
// products A_s B_s in one persistent launch (the attention backward's heads).
//
// Dual accumulators (dual = 1, column mode, 256-column tiles): each tile runs
// two products of the same shape, A B (k-blocks [0, k/2)) into TMEM columns
// [0, 256) and A2 B2 (k-blocks [k/2, k)) into [256, 512), and the epilogue
// reads both: the attention backward's scores Q K^T and dP = dO V^T for the
// same block, from which it makes P and dS together (EPI_DUAL_SOFTMAX).
//
// Stream-K (sk = 1): whole tiles dealt round-robin leave clusters idle in the
// last wave when the tile count is not a multiple of the cluster count.
// Here the whole waves stay as they are (concurrently running clusters share
// their operands in L2), and only the remainder tiles are split along K: the
// first clusters each run the head of one remainder tile and finish it, and
// the spare clusters run the remainder tiles' tails, laid end to end and cut
// evenly (sk_split).  A tail piece (a producer) stores its f32 partial
// accumulator to a workspace slot and publishes a flag; the head's cluster (the
// finisher) waits for those flags (bounded wait), adds the partials into its
// TMEM accumulator and runs the normal epilogue.  Producers never wait and a
// finisher piece is its cluster's last, so no wait can form a cycle; the grid
// is never larger than the clusters resident at once.  The partials are added
// in a fixed order, so results are run-to-run repeatable.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace tp {

constexpr int MAX_SHARDS = 8;

enum : int { ACT_NONE = 0, ACT_GELU_TANH = 1, ACT_GELU_ERF = 2, ACT_RELU = 3 };

// Kernel features, each compiled into its own instantiation so that the
// plain GEMM's loops carry none of the others' code: FEAT_BASE (whole tiles),
// FEAT_SK (stream-K), FEAT_DUAL (dual accumulators).
enum : int { FEAT_BASE = 0, FEAT_SK = 1, FEAT_DUAL = 2 };

template <int CG, bool WIDE = false, int FEAT = FEAT_BASE>
struct GemmCfg {
  static constexpr int BM = 128;                    // accumulator rows per CTA
  static constexpr int TILE_M = BM * CG;            // rows per (cluster) tile
  static constexpr int BN = 256;                    // columns per tile
  static constexpr int BK = 64;
#ifndef TP_GEMM_PAIR_STAGES
#define TP_GEMM_PAIR_STAGES 6
#endif
#ifndef TP_GEMM_L2_PREFETCH
#define TP_GEMM_L2_PREFETCH 0
#endif
#ifndef TP_GEMM_WIDE_STAGES
#define TP_GEMM_WIDE_STAGES 4
#endif
// bf16 epilogue chunks: both 32-column TMEM loads issued before one wait (1),
// or load-wait-convert per 32 columns (0).
#ifndef TP_GEMM_EPI_LD64
#define TP_GEMM_EPI_LD64 0
#endif
// Epilogue stores: each epilogue warp issues the TMA store of its own 32 rows
// (1), or one thread stores all 128 rows after a barrier of the four warps (0).
#ifndef TP_GEMM_WARP_STORES
#define TP_GEMM_WARP_STORES 0
#endif
  static_assert(!WIDE || CG == 2, "wide tiles need a CTA pair");
  // The dual-accumulator tiles have 4 k-blocks: fewer stages (5 for a pair,
  // 3 for a single CTA, whose B stage is twice as large), and the shared
  // memory that frees goes to a second pair of epilogue staging buffers.
  static constexpr int STAGES =
      FEAT == FEAT_DUAL ? (CG == 2 ? 5 : 3) : (WIDE ? TP_GEMM_WIDE_STAGES : (CG == 2 ? TP_GEMM_PAIR_STAGES : 4));
  static constexpr int PREFETCH = TP_GEMM_L2_PREFETCH;  // k-blocks ahead (0 = off)
  static constexpr int A_BYTES = BM * BK * 2;       // 16 KiB
  static constexpr int B_BOX_N = 64;                // 64 bf16 = one 128-byte swizzle row
  static constexpr int B_BOX_BYTES = BK * B_BOX_N * 2;  // 8 KiB
  static constexpr int B_COLS_CTA = BN / CG;        // B columns each CTA loads for the first MMA
  static constexpr int B_BOXES = B_COLS_CTA / B_BOX_N;
  static constexpr int B_REGION_BYTES = BK * B_COLS_CTA * 2;
  // Wide tiles: a second region holds this CTA's half of the second MMA's B.
  static constexpr int B_BYTES = (WIDE ? 2 : 1) * B_REGION_BYTES;
  static constexpr int ACC_BUFS = WIDE ? 1 : 2;     // accumulators in TMEM
  static constexpr int NUM_THREADS = 192;
  static constexpr int TMEM_COLS = 512;
  // Epilogue staging: buffers of 128 rows x 128 bytes (32 f32 or 64 bf16
  // columns), 128-byte swizzled, drained by TMA stores: two, used in turn;
  // four for the dual tiles (a P and a dS buffer, two pairs used in turn).
  static constexpr int EPI_BUF_BYTES = BM * 128;
  static constexpr int EPI_BUFS = FEAT == FEAT_DUAL ? 4 : 2;
  static constexpr int SMEM_BYTES =
      STAGES * (A_BYTES + B_BYTES) + EPI_BUFS * EPI_BUF_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(SMEM_BYTES <= 232448, "more dynamic shared memory than a CTA may have");
  static constexpr uint32_t IDESC = idesc_bf16_f32(TILE_M, BN, /*a_mn=*/false, /*b_mn=*/true);
  // B given K-major ([out, in] weights): one box of B_COLS_CTA rows x 64 k.
  static constexpr uint32_t IDESC_BK = idesc_bf16_f32(TILE_M, BN, /*a_mn=*/false, /*b_mn=*/false);
  // Narrow tiles (tile_n == 128, N-major B, not wide): one MMA of N = 128, for
  // which each CTA of a pair holds 64 B columns (one box).
  static constexpr int NARROW_N = 128;
  static constexpr uint32_t IDESC_N128 = idesc_bf16_f32(TILE_M, NARROW_N, /*a_mn=*/false, /*b_mn=*/true);
};

struct GemmArgs {
  // A [M, K] bf16 row-major, box {64, 128}: one map, or (a_per_shard, column
  // mode) one per shard, so that t independent products A_s B_s run in one launch.
  CUtensorMap tmA[MAX_SHARDS];
  CUtensorMap tmB[MAX_SHARDS];   // B shard s: [k rows, n cols] box {64, 64}, or K-major [n rows, k cols] box {64, BN/CG}
  // Output maps, 3-D {cols, M, splits}, box {128 B of columns, 128, 1}, 128-byte
  // swizzle: column mode one per shard (its column slice of C), row mode one.
  CUtensorMap tmC[MAX_SHARDS];
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
  int m_blocks, n_blocks, k_blocks;  // m_blocks counts TILE_M-row tiles
  // Tile order: 0, tile t is (m block t mod m_blocks, n block t / m_blocks),
  // so a wave shares B columns; 1, (t / n_blocks, t mod n_blocks), so a wave
  // shares A rows (for an A too large to stay in L2 across waves).
  int n_fastest;
  int act;
  int out_f32;
  // Split of the K loop into `splits` contiguous k-block ranges.  Work unit u
  // is (split u / tiles, tile u % tiles); split j writes its partial sum to
  // C + j * slot_stride (f32 only), and a later kernel adds the slots.
  int splits;
  long long slot_stride;
  int b_kmajor;                  // B shards stored [n, k] (nn.Linear [out, in] weights)
  int tile_n;                    // columns per tile: BN, or up to 2*BN for wide tiles
  int n2;                        // wide tiles: N of the second MMA (tile_n - BN), else 0
  uint32_t idesc2;               // wide tiles: instruction descriptor of the second MMA
  // A given M-major: the stored matrix is [K, M] (A^T of a row-major [M, K]),
  // loaded as two 64 x 64 boxes per CTA and read through an MN-major descriptor.
  int a_mnmajor;
  // Epilogue mode.  EPI_PLAIN: C = Act(acc).  EPI_AUX_PRE: also stores the
  // pre-activation acc (bf16) through tmAux (same tiling as C).  EPI_GRAD: bf16
  // C = acc * Act'(U), with U read from `aux` (bf16, row stride ld_aux, same
  // columns as C) — the backward of the activation fused into the GEMM.
  // EPI_SOFTMAX: bf16 C = 2^(acc * epi_scale - r), and EPI_DSOFTMAX: bf16
  // C = P (acc - r) epi_scale with P read from `aux` like U, where
  // r = rowvec[shard * rowvec_ld + row] (the softmax rebuilt from its log2
  // denominators, and its backward, fused into the attention backward's score
  // and dP GEMMs).
  int epi_mode;
  // Output rows split into shards of m_split_rows rows (0: off; a multiple
  // of the tile height): rows [s m_split_rows, (s+1) m_split_rows) go through
  // tmC[s] (its own buffer) at row offset 0 — the weight gradients G^T dZ of
  // all shards in one launch.
  int m_split_rows;
  CUtensorMap tmAux[MAX_SHARDS];
  const void* aux;
  long long ld_aux;
  int a_per_shard;
  const float* rowvec;
  long long rowvec_ld;
  float epi_scale;
  // Stream-K (see the top of this file).  sk_ws holds, per cluster c and CTA
  // rank r, a 128 x tile_n f32 block at ((c CG + r) 128 tile_n) (the partial a
  // producer piece leaves, float4 chunk j of row l at (j 128 + l)); sk_flags
  // [clusters x CG] hold the epoch of the last partial each one published.
  int sk;
  float* sk_ws;
  unsigned long long* sk_flags;
  unsigned long long sk_epoch;
  // Dual accumulators (see the top of this file): the second product's A and
  // B maps per shard, and its epilogue row vector and scale.
  int dual;
  CUtensorMap tmA2[MAX_SHARDS];
  CUtensorMap tmB2[MAX_SHARDS];
  const float* rowvec2;
  float epi_scale2;
};

enum : int { EPI_PLAIN = 0, EPI_AUX_PRE = 1, EPI_GRAD = 2, EPI_SOFTMAX = 3, EPI_DSOFTMAX = 4, EPI_DUAL_SOFTMAX = 5 };

// One piece of work of a cluster: the k-blocks [kb0, kb1) of a tile (of K
// split `split` in the K-split mode), and what its epilogue does with them;
// a stream-K producer piece's partial goes to workspace slot `slot`.
enum : int { ROLE_FULL = 0, ROLE_PRODUCER = 1, ROLE_FINISHER = 2 };
struct WorkItem {
  int tile, split, kb0, kb1, role, slot;
};

// Stream-K split of T tiles of kbt k-blocks over P clusters: W = T / P whole
// waves of tiles (dealt round-robin, so concurrently running clusters share
// operands in L2 as in the data-parallel schedule), then the R = T % P
// remaining tiles split along K: cluster c < R runs k-blocks [0, m) of
// remainder tile c (and finishes it), and the P - R spare clusters run the
// tails [m, kbt) of all R remainder tiles, laid end to end and cut into
// P - R equal ranges (producer pieces).  m = round(R kbt / P) balances the
// two.  m = 0 when there is no split (R == 0, or m would be 0 or kbt): the
// remainder tiles are then whole tiles too.
struct SkSplit {
  int W, R, m;
};

// The head takes SK_HEAD_EXTRA k-blocks more than the even share: a spare
// cluster's pieces each pay a partial-sum store and a pipeline restart.
constexpr int SK_HEAD_EXTRA = 3;
// Most producer pieces one remainder tile's tail may have (host plans that
// would exceed it keep whole tiles).
constexpr int SK_MAX_PRODUCERS = 16;

__host__ __device__ __forceinline__ SkSplit sk_split(long long T, int kbt, int P) {
  SkSplit s;
  s.W = static_cast<int>(T / P);
  s.R = static_cast<int>(T % P);
  const long long m = (2LL * s.R * kbt + P) / (2LL * P) + SK_HEAD_EXTRA;
  s.m = (s.R == 0 || m < 1 || m >= kbt) ? 0 : static_cast<int>(m);
  return s;
}

// The spare clusters whose tail ranges meet remainder tile r's tail
// [r L, (r+1) L) (L = kbt - m): written to list[0..n), in order; n <= max.
__host__ __device__ __forceinline__ int sk_producers(const SkSplit& sp, int kbt, int P, int r, int* list, int max) {
  const long long L = kbt - sp.m;
  const long long tt = static_cast<long long>(sp.R) * L;
  const long long spare = P - sp.R;
  const long long t0 = r * L, t1 = t0 + L;
  // first s with end > t0, last s with start < t1 (ends/starts floor(tt s / spare))
  long long s_lo = ((t0 + 1) * spare + tt - 1) / tt - 1;
  long long s_hi = (t1 * spare + tt - 1) / tt - 1;
  if (s_lo < 0) s_lo = 0;
  if (s_hi > spare - 1) s_hi = spare - 1;
  int n = 0;
  for (long long sc = s_lo; sc <= s_hi && n < max; ++sc) {
    const long long a = tt * sc / spare, b = tt * (sc + 1) / spare;
    if (b > a && a < t1 && b > t0) list[n++] = static_cast<int>(sc);
  }
  return n;
}

// Spare cluster s's range of the remainder tiles' tail k-blocks laid end to end.
__device__ __forceinline__ void sk_tail_range(const SkSplit& sp, int kbt, int P, int s, long long& a, long long& b) {
  const long long tt = static_cast<long long>(sp.R) * (kbt - sp.m);
  const int spare = P - sp.R;
  a = tt * s / spare;
  b = tt * (s + 1) / spare;
}

template <int FEAT>
__device__ __forceinline__ int num_work_items(const GemmArgs& p, int c, int nclusters) {
  const int num_tiles = p.m_blocks * p.n_blocks;
  if constexpr (FEAT != FEAT_SK) {
    const int units = num_tiles * p.splits;
    return c < units ? (units - 1 - c) / nclusters + 1 : 0;
  }
  const SkSplit sp = sk_split(num_tiles, p.k_blocks, nclusters);
  if (sp.R == 0) return sp.W;
  if (sp.m == 0) return sp.W + (c < sp.R ? 1 : 0);
  if (c < sp.R) return sp.W + 1;
  long long a, b;
  sk_tail_range(sp, p.k_blocks, nclusters, c - sp.R, a, b);
  const int L = p.k_blocks - sp.m;
  return sp.W + (b > a ? static_cast<int>((b - 1) / L - a / L + 1) : 0);
}

__device__ __forceinline__ void split_range(const GemmArgs& p, int split, int& kb0, int& kb1);

// The idx-th of cluster c's n work items, in processing order: its whole
// tiles first, then its remainder piece (a finisher, last) or its tail
// pieces (producers).
template <int FEAT>
__device__ __forceinline__ WorkItem work_item(const GemmArgs& p, int c, int nclusters, int idx, int n) {
  WorkItem w;
  w.split = 0;
  w.slot = 0;
  w.role = ROLE_FULL;
  const int num_tiles = p.m_blocks * p.n_blocks;
  if constexpr (FEAT != FEAT_SK) {
    const int unit = c + idx * nclusters;
    w.tile = unit % num_tiles;
    w.split = unit / num_tiles;
    split_range(p, w.split, w.kb0, w.kb1);
    return w;
  }
  (void)n;
  const SkSplit sp = sk_split(num_tiles, p.k_blocks, nclusters);
  w.kb0 = 0;
  w.kb1 = p.k_blocks;
  if (idx < sp.W) {
    w.tile = c + idx * nclusters;
    return w;
  }
  const int base = sp.W * nclusters;  // first remainder tile
  if (sp.m == 0) {
    w.tile = base + c;
    return w;
  }
  if (c < sp.R) {
    w.tile = base + c;
    w.kb1 = sp.m;
    w.role = ROLE_FINISHER;
    return w;
  }
  const int s = c - sp.R;
  const int L = p.k_blocks - sp.m;
  long long a, b;
  sk_tail_range(sp, p.k_blocks, nclusters, s, a, b);
  const int r = static_cast<int>(a / L) + (idx - sp.W);
  const long long lo = a > static_cast<long long>(r) * L ? a : static_cast<long long>(r) * L;
  const long long hi = b < static_cast<long long>(r + 1) * L ? b : static_cast<long long>(r + 1) * L;
  w.tile = base + r;
  w.kb0 = sp.m + static_cast<int>(lo - static_cast<long long>(r) * L);
  w.kb1 = sp.m + static_cast<int>(hi - static_cast<long long>(r) * L);
  w.role = ROLE_PRODUCER;
  w.slot = r + s;
  return w;
}

__device__ __forceinline__ void split_range(const GemmArgs& p, int split, int& kb0, int& kb1) {
  kb0 = static_cast<int>(static_cast<long long>(split) * p.k_blocks / p.splits);
  kb1 = static_cast<int>(static_cast<long long>(split + 1) * p.k_blocks / p.splits);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Epilogue work on one 128-byte output chunk of this thread's accumulator row:
// tcgen05.ld, activation, conversion, and a 128-byte-swizzled row write into
// the staging buffer.  The activation is a template argument so the element
// loop holds only that activation's instructions (a runtime switch per
// element gets if-converted into evaluating every activation).
template <int ACT>
__device__ __forceinline__ float act_t(float u) {
  if constexpr (ACT == ACT_GELU_TANH) {
    const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
    return 0.5f * u * (1.0f + tanh_fast(k0 * fmaf(0.044715f * u, u * u, u)));
  } else if constexpr (ACT == ACT_GELU_ERF) {
    return 0.5f * u * (1.0f + erff(u * 0.7071067811865476f));
  } else if constexpr (ACT == ACT_RELU) {
    return fmaxf(u, 0.0f);
  } else {
    return u;
  }
}

// d Act(u) / du for the backward epilogue (ReLU's derivative at 0 is 0).
template <int ACT>
__device__ __forceinline__ float act_grad_t(float u) {
  if constexpr (ACT == ACT_GELU_TANH) {
    const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
    const float t = tanh_fast(k0 * fmaf(0.044715f * u, u * u, u));
    return 0.5f * (1.0f + t) + 0.5f * u * (1.0f - t * t) * k0 * fmaf(3.0f * 0.044715f, u * u, 1.0f);
  } else if constexpr (ACT == ACT_GELU_ERF) {
    return 0.5f * (1.0f + erff(u * 0.7071067811865476f)) + u * 0.3989422804014327f * __expf(-0.5f * u * u);
  } else if constexpr (ACT == ACT_RELU) {
    return u > 0.0f ? 1.0f : 0.0f;
  } else {
    return 1.0f;
  }
}

// Backward epilogue chunk (bf16 out, 64 columns): acc * Act'(U) with this
// thread's U values read from global memory, 32 at a time (columns past
// `nvalid` and rows past M read nothing and use U = 0).
template <int ACT>
__device__ __forceinline__ void epi_chunk_grad(uint32_t taddr, uint8_t* stage_row, int row_local,
                                               const __nv_bfloat16* urow, int nvalid) {
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    float u[32];
    const int nv = nvalid - 32 * h;
    if (urow != nullptr && nv >= 32) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(urow + 32 * h) + j);
        const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(hv[e]);
          u[8 * j + 2 * e] = f.x;
          u[8 * j + 2 * e + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) u[j] = (urow != nullptr && j < nv) ? __bfloat162float(urow[32 * h + j]) : 0.0f;
    }
    uint32_t r[32];
    tmem_ld_32x32b_x32(taddr + h * 32, r);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i0 = 8 * j + 2 * e;
        w4[e] = pack_bf16x2(__uint_as_float(r[i0]) * act_grad_t<ACT>(u[i0]),
                            __uint_as_float(r[i0 + 1]) * act_grad_t<ACT>(u[i0 + 1]));
      }
      *reinterpret_cast<uint4*>(stage_row + (((4 * h + j) ^ (row_local & 7)) << 4)) =
          make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  }
}

// Softmax epilogue chunk (bf16 out, 64 columns): 2^(acc * scale - r).
__device__ __forceinline__ void epi_chunk_softmax(uint32_t taddr, uint8_t* stage_row, int row_local, float r,
                                                  float scale) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(taddr + h * 32, v);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i0 = 8 * j + 2 * e;
        w4[e] = pack_bf16x2(exp2f(fmaf(__uint_as_float(v[i0]), scale, -r)),
                            exp2f(fmaf(__uint_as_float(v[i0 + 1]), scale, -r)));
      }
      *reinterpret_cast<uint4*>(stage_row + (((4 * h + j) ^ (row_local & 7)) << 4)) =
          make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  }
}

// Softmax-backward epilogue chunk (bf16 out, 64 columns): P (acc - r) scale.
// The chunk's 64 P values (bf16 pairs) are loaded first, all eight 16-byte
// loads in flight at once (columns past `nvalid` and rows past M use P = 0).
__device__ __forceinline__ void epi_load_p64(const __nv_bfloat16* prow, int nvalid, uint32_t (&pw)[32]) {
  if (prow != nullptr && nvalid >= 64) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(prow) + j);
      pw[4 * j] = w.x;
      pw[4 * j + 1] = w.y;
      pw[4 * j + 2] = w.z;
      pw[4 * j + 3] = w.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float lo = (prow != nullptr && 2 * j < nvalid) ? __bfloat162float(prow[2 * j]) : 0.0f;
      const float hi = (prow != nullptr && 2 * j + 1 < nvalid) ? __bfloat162float(prow[2 * j + 1]) : 0.0f;
      pw[j] = pack_bf16x2(lo, hi);
    }
  }
}

__device__ __forceinline__ void epi_chunk_dsoftmax(uint32_t taddr, uint8_t* stage_row, int row_local,
                                                   const uint32_t (&pw)[32], float r, float scale) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(taddr + h * 32, v);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i0 = 8 * j + 2 * e;  // columns 32 h + i0, i0 + 1 = bf16 pair 16 h + 4 j + e
        const uint32_t pp = pw[16 * h + 4 * j + e];
        const float2 pf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pp));
        w4[e] = pack_bf16x2(pf.x * (__uint_as_float(v[i0]) - r) * scale,
                            pf.y * (__uint_as_float(v[i0 + 1]) - r) * scale);
      }
      *reinterpret_cast<uint4*>(stage_row + (((4 * h + j) ^ (row_local & 7)) << 4)) =
          make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  }
}

// Dual softmax epilogue chunk (bf16 out, 64 columns): from the scores s (TMEM
// columns taddr ..) and dP (taddr + 256 ..) of the same row,
//   P  = 2^(s * scale1 - r1)                 into stage_p,
//   dS = P (dP - r2) scale2                  into stage_ds,
// with P in f32 for dS (its bf16 rounding only for the stored copy).
__device__ __forceinline__ void epi_chunk_dual_softmax(uint32_t taddr, uint8_t* stage_p, uint8_t* stage_ds,
                                                       int row_local, float r1, float scale1, float r2,
                                                       float scale2) {
  // P = 2^(s scale1 - r1) with the forward softmax's exponential (ex2.approx,
  // so P is rebuilt as the forward made it), dS = (P (dp - r2)) scale2; the
  // arithmetic on f32 pairs (f32x2), two columns per instruction.
  const unsigned long long sc = f2_pack(scale1, scale1), nr = f2_pack(-r1, -r1);
  const unsigned long long d2 = f2_pack(r2, r2), s2 = f2_pack(scale2, scale2);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t sv[32], dv[32];
    tmem_ld_32x32b_x32(taddr + h * 32, sv);
    tmem_ld_32x32b_x32(taddr + 256 + h * 32, dv);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t wp[4], wd[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i0 = 8 * j + 2 * e;
        float x0, x1, q0, q1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[i0]), __uint_as_float(sv[i0 + 1])), sc, nr), x0, x1);
        const float p0 = exp2_fast(x0), p1 = exp2_fast(x1);
        wp[e] = pack_bf16x2(p0, p1);
        const unsigned long long g =
            f2_sub(f2_pack(__uint_as_float(dv[i0]), __uint_as_float(dv[i0 + 1])), d2);
        f2_unpack(f2_mul(f2_mul(f2_pack(p0, p1), g), s2), q0, q1);
        wd[e] = pack_bf16x2(q0, q1);
      }
      const int off = ((4 * h + j) ^ (row_local & 7)) << 4;
      *reinterpret_cast<uint4*>(stage_p + off) = make_uint4(wp[0], wp[1], wp[2], wp[3]);
      *reinterpret_cast<uint4*>(stage_ds + off) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
    }
  }
}

template <int ACT>
__device__ __forceinline__ void epi_chunk_f32(uint32_t taddr, uint8_t* stage_row, int row_local) {
  uint32_t r[32];
  tmem_ld_32x32b_x32(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 8; ++j) {  // 16-byte chunk j = 4 f32
    uint4 w;
    w.x = __float_as_uint(act_t<ACT>(__uint_as_float(r[4 * j + 0])));
    w.y = __float_as_uint(act_t<ACT>(__uint_as_float(r[4 * j + 1])));
    w.z = __float_as_uint(act_t<ACT>(__uint_as_float(r[4 * j + 2])));
    w.w = __float_as_uint(act_t<ACT>(__uint_as_float(r[4 * j + 3])));
    *reinterpret_cast<uint4*>(stage_row + ((j ^ (row_local & 7)) << 4)) = w;
  }
}

template <int ACT>
__device__ __forceinline__ void epi_chunk_bf16(uint32_t taddr, uint8_t* stage_row, int row_local) {
#if TP_GEMM_EPI_LD64
  // Both 32-column loads in flight before one wait.
  uint32_t r2[2][32];
  tmem_ld_32x32b_x32(taddr, r2[0]);
  tmem_ld_32x32b_x32(taddr + 32, r2[1]);
  tmem_wait_ld();
#endif
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#if TP_GEMM_EPI_LD64
    const uint32_t (&r)[32] = r2[h];
#else
    uint32_t r[32];
    tmem_ld_32x32b_x32(taddr + h * 32, r);
    tmem_wait_ld();
#endif
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // 16-byte chunk 4h+j = 8 bf16
      uint4 w;
      w.x = pack_bf16x2(act_t<ACT>(__uint_as_float(r[8 * j + 0])), act_t<ACT>(__uint_as_float(r[8 * j + 1])));
      w.y = pack_bf16x2(act_t<ACT>(__uint_as_float(r[8 * j + 2])), act_t<ACT>(__uint_as_float(r[8 * j + 3])));
      w.z = pack_bf16x2(act_t<ACT>(__uint_as_float(r[8 * j + 4])), act_t<ACT>(__uint_as_float(r[8 * j + 5])));
      w.w = pack_bf16x2(act_t<ACT>(__uint_as_float(r[8 * j + 6])), act_t<ACT>(__uint_as_float(r[8 * j + 7])));
      *reinterpret_cast<uint4*>(stage_row + (((4 * h + j) ^ (row_local & 7)) << 4)) = w;
    }
  }
}

template <int ACT>
__device__ __forceinline__ void epi_chunk(bool out_f32, uint32_t taddr, uint8_t* stage_row, int row_local) {
  if (out_f32) epi_chunk_f32<ACT>(taddr, stage_row, row_local);
  else epi_chunk_bf16<ACT>(taddr, stage_row, row_local);
}

// Tile coordinates shared by the three roles.
struct TileCoord {
  int m0;        // first row of the (cluster) tile
  int shard;     // column mode: shard owning the tile's columns
  int n_in;      // first column inside the B operand (shard-local in column mode)
  int out_col0;  // first column of C
  int n_valid;   // valid columns in this tile (<= BN)
};

template <int CG>
__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& p, int tile) {
  using C = GemmCfg<CG>;
  TileCoord c;
  const int mb = p.n_fastest ? tile / p.n_blocks : tile % p.m_blocks;
  const int nb = p.n_fastest ? tile % p.n_blocks : tile / p.m_blocks;
  c.m0 = mb * C::TILE_M;
  if (!p.row_mode) {
    c.shard = nb / p.n_blocks_per_shard;
    c.n_in = (nb % p.n_blocks_per_shard) * p.tile_n;
    c.out_col0 = c.shard * p.shard_n + c.n_in;
  } else {
    c.shard = 0;
    c.n_in = nb * p.tile_n;
    c.out_col0 = c.n_in;
  }
  c.n_valid = min(p.tile_n, p.shard_n - c.n_in);
  return c;
}

// Shard, A column and B row of k-block kb.
template <int FEAT = FEAT_BASE>
__device__ __forceinline__ void kblock_coords(const GemmArgs& p, const TileCoord& tc, int kb, int& shard, int& a_x,
                                              int& b_y) {
  constexpr int BK = 64;
  if (FEAT == FEAT_DUAL) {  // k-blocks [k/2, k) are the second product's, from its own k = 0
    const int half = p.k_blocks / 2;
    shard = tc.shard;
    b_y = (kb < half ? kb : kb - half) * BK;
    a_x = b_y;
    return;
  }
  if (p.row_mode) {
    shard = kb / p.k_blocks_per_shard;
    b_y = (kb % p.k_blocks_per_shard) * BK;
    a_x = shard * p.shard_k + b_y;
  } else {
    shard = tc.shard;
    b_y = kb * BK;
    a_x = b_y;
  }
}

// Number of 64-column B boxes CTA `rank` of the pair loads for a tile (N-major
// B); a K-major B is one box of B_COLS_CTA rows, counted here as B_BOXES.
// Narrow tiles: B columns per CTA are NARROW_N / CG (a pair: one box each).
template <int CG>
__device__ __forceinline__ int b_boxes_for(int n_valid, int rank, int b_kmajor, bool narrow = false) {
  using C = GemmCfg<CG>;
  const int per_cta = narrow ? C::NARROW_N / CG : C::B_COLS_CTA;
  const int cols = min(n_valid, narrow ? C::NARROW_N : C::BN) - rank * per_cta;
  if (cols <= 0) return 0;
  if (b_kmajor) return C::B_BOXES;
  return min(per_cta / C::B_BOX_N, (cols + C::B_BOX_N - 1) / C::B_BOX_N);
}

// Narrow tiles: 128-column tiles with an N-major B run one N = 128 MMA.
template <bool WIDE>
__device__ __forceinline__ bool narrow_tiles(const GemmArgs& p) {
  return !WIDE && p.tile_n == 128 && !p.b_kmajor;
}

// A bytes a CTA whose rows start at row0 brings into a stage: one 128 x 64
// K-major box, or (M-major A) one 64 x 64 box per 64 rows that exist.
__device__ __forceinline__ int a_mn_boxes(const GemmArgs& p, int row0) {
  const int rows = p.M - row0;
  return rows <= 0 ? 0 : (rows >= 128 ? 2 : (rows + 63) / 64);
}
__device__ __forceinline__ uint32_t a_bytes_for(const GemmArgs& p, int row0) {
  if (p.a_mnmajor) return static_cast<uint32_t>(a_mn_boxes(p, row0)) * 8192u;
  return row0 < p.M ? 16384u : 0u;
}

// Wide tiles: B boxes CTA `rank` loads for the second MMA, whose n2 columns
// (tile columns [BN, BN + n2)) the pair splits in halves of n2/2.  Counted in
// B_BOX_BYTES units; a K-major B is one box of up to B_COLS_CTA rows.
__device__ __forceinline__ int b2_boxes_for(int n_valid, int n2, int rank, int b_kmajor) {
  using C = GemmCfg<2, true>;
  const int half = n2 / 2;
  const int cols = min(n_valid - C::BN - rank * half, half);
  if (cols <= 0) return 0;
  if (b_kmajor) return C::B_BOXES;
  return (cols + C::B_BOX_N - 1) / C::B_BOX_N;
}

template <int CG, bool WIDE = false, int FEAT = FEAT_BASE>
__global__ void __launch_bounds__(GemmCfg<CG>::NUM_THREADS, 1) gemm_tcgen05_kernel(const __grid_constant__ GemmArgs p) {
  using C = GemmCfg<CG, WIDE, FEAT>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_BYTES;
  uint8_t* sEpi = sB + STAGES * C::B_BYTES;  // EPI_BUFS x EPI_BUF_BYTES
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + C::EPI_BUFS * C::EPI_BUF_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], CG == 2 ? 4 * CG : 128);
    }
    mbar_init(drain, 1);
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < (p.a_per_shard ? p.t : 1); ++s) tma_prefetch_desc(&p.tmA[s]);
    for (int s = 0; s < p.t; ++s) tma_prefetch_desc(&p.tmB[s]);
  }
  if (warp == 2 && lane == 0) {
    for (int s = 0; s < (p.row_mode ? 1 : p.t); ++s) tma_prefetch_desc(&p.tmC[s]);
  }
  if (warp == 1) {
    tmem_alloc<CG>(tmem_holder, C::TMEM_COLS);
    tmem_relinquish<CG>();
  }
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync();
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // The prologue above touched no global memory: only now wait for the
  // preceding kernel (whose output may be A, or whose inputs C may overwrite),
  // and let the next kernel start its own prologue as SMs free up.
  griddep_wait();
  griddep_launch_dependents();

  const bool narrow = narrow_tiles<WIDE>(p);
  const int cluster_id = blockIdx.x / CG;
  const int num_clusters = gridDim.x / CG;
  const int num_items = num_work_items<FEAT>(p, cluster_id, num_clusters);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int armed[STAGES];  // parity of the last phase this thread armed per stage (leader)
#pragma unroll
      for (int s = 0; s < STAGES; ++s) armed[s] = -1;
      for (int idx = 0; idx < num_items && ok; ++idx) {
        const WorkItem wi = work_item<FEAT>(p, cluster_id, num_clusters, idx, num_items);
        const int kb_begin = wi.kb0, kb_end = wi.kb1;
        const TileCoord tc = tile_coord<CG>(p, wi.tile);
        const CUtensorMap* mA = &p.tmA[p.a_per_shard ? tc.shard : 0];
        const int my_row0 = tc.m0 + static_cast<int>(rank) * C::BM;
        const bool my_a = my_row0 < p.M;
        const int my_aboxes = a_mn_boxes(p, my_row0);  // M-major A: 64-row boxes this CTA loads
        const int my_boxes = b_boxes_for<CG>(tc.n_valid, rank, p.b_kmajor, narrow);
        const int my_boxes2 = WIDE ? b2_boxes_for(tc.n_valid, p.n2, rank, p.b_kmajor) : 0;
        uint32_t bytes = 0;  // leader: bytes the whole tile stage brings in
        for (int r = 0; r < CG; ++r) {
          bytes += a_bytes_for(p, tc.m0 + r * C::BM) + b_boxes_for<CG>(tc.n_valid, r, p.b_kmajor, narrow) * C::B_BOX_BYTES;
          if constexpr (WIDE) bytes += b2_boxes_for(tc.n_valid, p.n2, r, p.b_kmajor) * C::B_BOX_BYTES;
        }
        const int b_x0 = tc.n_in + static_cast<int>(rank) * (narrow ? C::NARROW_N / CG : C::B_COLS_CTA);
        const int b_x2 = tc.n_in + C::BN + static_cast<int>(rank) * (p.n2 / 2);  // wide: second region
        for (int kb = kb_begin; kb < kb_end; ++kb) {
          if constexpr (C::PREFETCH > 0) {
            const int kp = kb + C::PREFETCH;
            if (kp < kb_end && !p.a_mnmajor) {
              int ps, pa, pb;
              kblock_coords<FEAT>(p, tc, kp, ps, pa, pb);
              const bool second = FEAT == FEAT_DUAL && kp >= p.k_blocks / 2;
              const CUtensorMap* pA = second ? &p.tmA2[p.a_per_shard ? tc.shard : 0] : mA;
              const CUtensorMap* pB = second ? &p.tmB2[ps] : &p.tmB[ps];
              if (my_a) tma_prefetch_l2_2d(pA, pa, my_row0);
              for (int j = 0; j < my_boxes; ++j) tma_prefetch_l2_2d(pB, b_x0 + j * C::B_BOX_N, pb);
            }
          }
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          int shard, a_x, b_y;
          kblock_coords<FEAT>(p, tc, kb, shard, a_x, b_y);
          uint8_t* dA = sA + stage * C::A_BYTES;
          uint8_t* dB = sB + stage * C::B_BYTES;
          // Dual accumulators: the second half of the k-blocks is the second product's.
          const bool second = FEAT == FEAT_DUAL && kb >= p.k_blocks / 2;
          const CUtensorMap* mAk = second ? &p.tmA2[p.a_per_shard ? tc.shard : 0] : mA;
          const CUtensorMap* mBk = second ? &p.tmB2[shard] : &p.tmB[shard];
          if constexpr (CG == 1) {
            mbar_arrive_expect_tx(&full[stage], bytes);
            armed[stage] = static_cast<int>(phase);
            if (p.a_mnmajor) {
              for (int j = 0; j < my_aboxes; ++j)
                tma_load_2d(dA + j * C::B_BOX_BYTES, mAk, my_row0 + j * 64, a_x, &full[stage]);
            } else {
              tma_load_2d(dA, mAk, a_x, my_row0, &full[stage]);
            }
            if (p.b_kmajor) {
              if (my_boxes) tma_load_2d(dB, mBk, b_y, b_x0, &full[stage]);
            } else {
              for (int j = 0; j < my_boxes; ++j)
                tma_load_2d(dB + j * C::B_BOX_BYTES, mBk, b_x0 + j * C::B_BOX_N, b_y, &full[stage]);
            }
          } else {
            const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
            if (leader) {
              mbar_arrive_expect_tx(&full[stage], bytes);
              armed[stage] = static_cast<int>(phase);
            }
            if (p.a_mnmajor) {
              for (int j = 0; j < my_aboxes; ++j)
                tma_load_2d_pair(dA + j * C::B_BOX_BYTES, mAk, my_row0 + j * 64, a_x, bar);
            } else if (my_a) {
              tma_load_2d_pair(dA, mAk, a_x, my_row0, bar);
            }
            if (p.b_kmajor) {
              if (my_boxes) tma_load_2d_pair(dB, mBk, b_y, b_x0, bar);
            } else {
              for (int j = 0; j < my_boxes; ++j)
                tma_load_2d_pair(dB + j * C::B_BOX_BYTES, mBk, b_x0 + j * C::B_BOX_N, b_y, bar);
            }
            if constexpr (WIDE) {
              uint8_t* dB2 = dB + C::B_REGION_BYTES;
              if (p.b_kmajor) {
                if (my_boxes2) tma_load_2d_pair(dB2, mBk, b_y, b_x2, bar);
              } else {
                for (int j = 0; j < my_boxes2; ++j)
                  tma_load_2d_pair(dB2 + j * C::B_BOX_BYTES, mBk, b_x2 + j * C::B_BOX_N, b_y, bar);
              }
            }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // Let every copy this CTA's barriers still expect land before exit.
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
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      constexpr int acc_bufs = FEAT == FEAT_DUAL ? 1 : C::ACC_BUFS;  // dual: both 256-column halves per tile
      for (int idx = 0; idx < num_items && ok; ++idx) {
        const WorkItem wi = work_item<FEAT>(p, cluster_id, num_clusters, idx, num_items);
        const int kb_begin = wi.kb0, kb_end = wi.kb1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
        // Wide tiles: the second MMA only where the tile has columns past BN.
        const bool two = WIDE && tile_coord<CG>(p, wi.tile).n_valid > C::BN;
        for (int kb = kb_begin; kb < kb_end; ++kb) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
          const uint32_t idesc = (narrow ? C::IDESC_N128 : (p.b_kmajor ? C::IDESC_BK : C::IDESC)) |
                                 (p.a_mnmajor ? (1u << 15) : 0u);
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            // A K-major: 16 k-elements = 32 bytes further along the swizzled row.
            // A M-major: like an N-major B (64-row chunks 8 KiB apart).
            const uint64_t ad = p.a_mnmajor ? sdesc_sw128(a0 + kk * 2048, C::B_BOX_BYTES, 1024)
                                            : sdesc_sw128(a0 + kk * 32, 16, 1024);
            // B N-major: 16 k-rows = 2 x (8 rows x 128 B) further; 64-column
            // chunks are B_BOX_BYTES apart (leading offset), 8-row groups 1 KiB.
            // B K-major: like A.
            const uint64_t bd = p.b_kmajor ? sdesc_sw128(b0 + kk * 32, 16, 1024)
                                           : sdesc_sw128(b0 + kk * 2048, C::B_BOX_BYTES, 1024);
            uint32_t accum = (kb != kb_begin || kk != 0) ? 1u : 0u;
            uint32_t dt = d_tmem;
            if constexpr (FEAT == FEAT_DUAL) {
              const bool second = kb >= p.k_blocks / 2;
              if (kb == p.k_blocks / 2 && kk == 0) accum = 0u;  // the second product starts its own sum
              if (second) dt += static_cast<uint32_t>(C::BN);
            }
            if constexpr (CG == 1) umma_bf16(dt, ad, bd, idesc, accum);
            else umma_bf16_pair(dt, ad, bd, idesc, accum);
            if constexpr (WIDE) {
              if (two) {
                const uint32_t b2 = b0 + C::B_REGION_BYTES;
                const uint64_t bd2 = p.b_kmajor ? sdesc_sw128(b2 + kk * 32, 16, 1024)
                                                : sdesc_sw128(b2 + kk * 2048, C::B_BOX_BYTES, 1024);
                umma_bf16_pair(d_tmem + C::BN, ad, bd2, p.idesc2, accum);
              }
            }
          }
          if constexpr (CG == 1) umma_commit(&empty[stage]);
          else umma_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if constexpr (CG == 1) umma_commit(&tfull[acc]);
        else umma_commit_pair_mc(&tfull[acc], 0x3);
        if (++acc == acc_bufs) { acc = 0; acc_phase ^= 1; }
      }
      if (!ok) {
        // Wait (bounded) for every MMA already issued before TMEM is freed.
        if constexpr (CG == 1) umma_commit(drain);
        else umma_commit_pair_mc(drain, 0x1);
        const uint32_t a = smem_u32(drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(a, 0) && clock64() - t0 < WAIT_LIMIT_CYCLES) {}
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Per 128-byte column chunk: tcgen05.ld of this thread's accumulator row,
    // activation, conversion, a swizzled row write into a staging buffer, then
    // one TMA store of the 128 x chunk box (double-buffered).  TMA clips rows
    // beyond M and columns beyond the shard / output width.
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_local = q * 32 + lane;
    const bool elected = threadIdx.x == 64;
    const int cw = p.out_f32 ? 32 : 64;  // columns per 128-byte chunk
    int acc = 0;
    uint32_t acc_phase = 0;
    int buf = 0;
    const uint32_t tempty_leader0 = CG == 2 ? mapa_shared(smem_u32(&tempty[0]), 0) : 0u;
    constexpr int acc_bufs = FEAT == FEAT_DUAL ? 1 : C::ACC_BUFS;
    for (int idx = 0; idx < num_items; ++idx) {
      const WorkItem wi = work_item<FEAT>(p, cluster_id, num_clusters, idx, num_items);
      const TileCoord tc = tile_coord<CG>(p, wi.tile);
      const int split = wi.split;
      const int y0 = tc.m0 + static_cast<int>(rank) * C::BM;
      const int mshard = p.m_split_rows ? tc.m0 / p.m_split_rows : 0;
      const int ystore = y0 - mshard * p.m_split_rows;
      const CUtensorMap* tmC = &p.tmC[p.m_split_rows ? mshard : (p.row_mode ? 0 : tc.shard)];
      const CUtensorMap* tmAux = &p.tmAux[p.row_mode ? 0 : tc.shard];
      // All 128 epilogue threads take the same decision (they meet at named
      // barriers below).
      if (!named_barrier_and(1, 128, mbar_wait(&tfull[acc], acc_phase))) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * C::BN);
      if (FEAT == FEAT_SK && wi.role == ROLE_PRODUCER) {
        // Stream-K producer piece: the raw f32 accumulator goes to this CTA's
        // block of the workspace (coalesced: float4 chunk j of row l at
        // j * 128 + l), then the TMEM buffer is handed back and the flag
        // published once every thread's stores are visible.
        float4* dst = reinterpret_cast<float4*>(p.sk_ws + static_cast<long long>(wi.slot * CG + rank) * C::BM *
                                                              p.tile_n) + row_local;
        for (int c32 = 0; c32 < p.tile_n / 32; ++c32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_row + c32 * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            __stcg(dst + static_cast<long long>(c32 * 8 + j) * C::BM,
                   make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                               __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
        }
        tc_fence_before();
        if constexpr (CG == 1) {
          mbar_arrive(&tempty[acc]);
        } else {
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty_leader0 + static_cast<uint32_t>(acc * sizeof(uint64_t)));
        }
        __threadfence();
        named_barrier_sync(1, 128);
        if (elected) flag_publish(p.sk_flags + wi.slot * CG + rank, p.sk_epoch);
        if (++acc == acc_bufs) { acc = 0; acc_phase ^= 1; }
        continue;
      }
      if (FEAT == FEAT_SK && wi.role == ROLE_FINISHER) {
        // Stream-K finisher piece: wait for every producer piece of this
        // remainder tile's tail (the spare clusters whose tail ranges meet
        // it, listed once), then add their partials into the TMEM accumulator
        // in the spare clusters' order.
        const SkSplit sp = sk_split(static_cast<long long>(p.m_blocks) * p.n_blocks, p.k_blocks, num_clusters);
        const int r = wi.tile - sp.W * num_clusters;
        int prod[SK_MAX_PRODUCERS];
        const int nprod = sk_producers(sp, p.k_blocks, num_clusters, r, prod, SK_MAX_PRODUCERS);
        if (elected) {
          for (int i = 0; i < nprod; ++i)
            if (!flag_wait_eq(p.sk_flags + (r + prod[i]) * CG + rank, p.sk_epoch)) break;
        }
        named_barrier_sync(1, 128);
        for (int c32 = 0; c32 < p.tile_n / 32; ++c32) {
          uint32_t rr[32];
          tmem_ld_32x32b_x32(t_row + c32 * 32, rr);
          tmem_wait_ld();
          for (int i = 0; i < nprod; ++i) {
            const float4* src = reinterpret_cast<const float4*>(
                                    p.sk_ws + static_cast<long long>((r + prod[i]) * CG + rank) * C::BM * p.tile_n) +
                                row_local;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 v = __ldcg(src + static_cast<long long>(c32 * 8 + j) * C::BM);
              rr[4 * j] = __float_as_uint(__uint_as_float(rr[4 * j]) + v.x);
              rr[4 * j + 1] = __float_as_uint(__uint_as_float(rr[4 * j + 1]) + v.y);
              rr[4 * j + 2] = __float_as_uint(__uint_as_float(rr[4 * j + 2]) + v.z);
              rr[4 * j + 3] = __float_as_uint(__uint_as_float(rr[4 * j + 3]) + v.w);
            }
          }
          tmem_st_32x32b_x32(t_row + c32 * 32, rr);
        }
        tmem_wait_st();
      }
      const int nchunks = (tc.n_valid + cw - 1) / cw;
      const int parts = p.epi_mode == EPI_AUX_PRE ? 2 : 1;  // aux (pre-activation) store first
      const int grow = y0 + row_local;
      const float rv = (p.rowvec != nullptr && grow < p.M)
                           ? __ldg(p.rowvec + static_cast<long long>(tc.shard) * p.rowvec_ld + grow)
                           : 0.0f;
      if constexpr (FEAT == FEAT_DUAL) {
        // P into staging buffer 2b and dS into 2b + 1, then one store of
        // each (one bulk group); the pairs b = 0, 1 are used in turn, so a
        // chunk is computed while the previous chunk's stores drain.
        const float rv2 = (p.rowvec2 != nullptr && grow < p.M)
                              ? __ldg(p.rowvec2 + static_cast<long long>(tc.shard) * p.rowvec_ld + grow)
                              : 0.0f;
        for (int c = 0; c < nchunks; ++c) {
          uint8_t* sP = sEpi + (2 * buf) * C::EPI_BUF_BYTES;
          uint8_t* sDS = sP + C::EPI_BUF_BYTES;
#if TP_GEMM_WARP_STORES
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
#else
          if (elected) bulk_wait_group_read<1>();
          named_barrier_sync(1, 128);
#endif
          epi_chunk_dual_softmax(t_row + c * 64, sP + row_local * 128, sDS + row_local * 128, row_local, rv,
                                 p.epi_scale, rv2, p.epi_scale2);
          if (c == nchunks - 1) {
            tc_fence_before();
            if constexpr (CG == 1) {
              mbar_arrive(&tempty[acc]);
            } else {
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster(tempty_leader0 + static_cast<uint32_t>(acc * sizeof(uint64_t)));
            }
          }
          fence_proxy_async_smem();
#if TP_GEMM_WARP_STORES
          __syncwarp();
          if (lane == 0 && y0 + q * 32 < p.M) {
            tma_store_3d(tmC, sP + q * 32 * 128, tc.n_in + c * 64, ystore + q * 32, 0);
            tma_store_3d(tmAux, sDS + q * 32 * 128, tc.n_in + c * 64, ystore + q * 32, 0);
          }
          if (lane == 0) bulk_commit_group();  // an empty group keeps the count of groups per pair
#else
          named_barrier_sync(1, 128);
          if (elected) {
            if (y0 < p.M) {
              tma_store_3d(tmC, sP, tc.n_in + c * 64, ystore, 0);
              tma_store_3d(tmAux, sDS, tc.n_in + c * 64, ystore, 0);
            }
            bulk_commit_group();
          }
#endif
          buf ^= 1;
        }
      } else {
        for (int c = 0; c < nchunks; ++c) {
          for (int part = 0; part < parts; ++part) {
            // The TMA store that last read this staging buffer must be done with it.
#if TP_GEMM_WARP_STORES
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
#else
            if (elected) bulk_wait_group_read<1>();
            named_barrier_sync(1, 128);
#endif
            uint8_t* stage_row = sEpi + buf * C::EPI_BUF_BYTES + row_local * 128;
            const uint32_t taddr = t_row + c * (p.out_f32 ? 32 : 64);
            if (p.epi_mode == EPI_SOFTMAX) {
              epi_chunk_softmax(taddr, stage_row, row_local, rv, p.epi_scale);
            } else if (p.epi_mode == EPI_DSOFTMAX) {
              const __nv_bfloat16* prow =
                  grow < p.M ? static_cast<const __nv_bfloat16*>(p.aux) + static_cast<long long>(grow) * p.ld_aux +
                                   tc.out_col0 + c * 64
                             : nullptr;
              uint32_t pw[32];
              epi_load_p64(prow, tc.n_valid - c * 64, pw);
              epi_chunk_dsoftmax(taddr, stage_row, row_local, pw, rv, p.epi_scale);
            } else if (p.epi_mode == EPI_GRAD) {
              const __nv_bfloat16* urow =
                  grow < p.M ? static_cast<const __nv_bfloat16*>(p.aux) + static_cast<long long>(grow) * p.ld_aux +
                                   tc.out_col0 + c * 64
                             : nullptr;
              const int nvalid = tc.n_valid - c * 64;
              switch (p.act) {  // uniform: one branch per chunk
                case ACT_GELU_TANH: epi_chunk_grad<ACT_GELU_TANH>(taddr, stage_row, row_local, urow, nvalid); break;
                case ACT_GELU_ERF: epi_chunk_grad<ACT_GELU_ERF>(taddr, stage_row, row_local, urow, nvalid); break;
                case ACT_RELU: epi_chunk_grad<ACT_RELU>(taddr, stage_row, row_local, urow, nvalid); break;
                default: epi_chunk_grad<ACT_NONE>(taddr, stage_row, row_local, urow, nvalid); break;
              }
            } else if (part < parts - 1) {
              epi_chunk<ACT_NONE>(p.out_f32, taddr, stage_row, row_local);
            } else {
              switch (p.act) {  // uniform: one branch per chunk
                case ACT_GELU_TANH: epi_chunk<ACT_GELU_TANH>(p.out_f32, taddr, stage_row, row_local); break;
                case ACT_GELU_ERF: epi_chunk<ACT_GELU_ERF>(p.out_f32, taddr, stage_row, row_local); break;
                case ACT_RELU: epi_chunk<ACT_RELU>(p.out_f32, taddr, stage_row, row_local); break;
                default: epi_chunk<ACT_NONE>(p.out_f32, taddr, stage_row, row_local); break;
              }
            }
            if (c == nchunks - 1 && part == parts - 1) {
              // Every accumulator column of this tile has been read: hand the
              // TMEM buffer back to the MMA issuer before the last store.
              tc_fence_before();
              if constexpr (CG == 1) {
                mbar_arrive(&tempty[acc]);
              } else {
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(tempty_leader0 + static_cast<uint32_t>(acc * sizeof(uint64_t)));
              }
            }
            fence_proxy_async_smem();
#if TP_GEMM_WARP_STORES
            // Each warp stores its own 32 rows (a 4 KiB, 1 KiB-aligned slice of the
            // staging buffer, so the 128-byte swizzle pattern is the same).
            __syncwarp();
            if (lane == 0 && y0 + q * 32 < p.M) {
              const CUtensorMap* map = part < parts - 1 ? tmAux : tmC;
              tma_store_3d(map, sEpi + buf * C::EPI_BUF_BYTES + q * 32 * 128, tc.n_in + c * cw, ystore + q * 32, split);
              bulk_commit_group();
            }
#else
            named_barrier_sync(1, 128);
            if (elected && y0 < p.M) {
              const CUtensorMap* map = part < parts - 1 ? tmAux : tmC;
              tma_store_3d(map, sEpi + buf * C::EPI_BUF_BYTES, tc.n_in + c * cw, ystore, split);
              bulk_commit_group();
            }
#endif
            buf ^= 1;
          }
        }
      }
      if (++acc == acc_bufs) { acc = 0; acc_phase ^= 1; }
    }
#if TP_GEMM_WARP_STORES
    if (lane == 0) bulk_wait_group_all();
#else
    if (elected) bulk_wait_group_all();
#endif
  }

  tc_fence_before();
  if constexpr (CG == 2) cluster_sync();
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<CG>(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace tp
