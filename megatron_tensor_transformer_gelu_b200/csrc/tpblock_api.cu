// C ABI of the tensor-parallel sublayer library (declared in include/tpblock.h).
//
// Host side only: argument checks, workspace carving, TMA tensor-map encoding,
// launch sequencing on the caller's stream, optional per-kernel event timing.
// Every step of the computation runs in this library's kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <chrono>
#include <mutex>
#include <utility>

#include "../../include/tpblock.h"
#include "attention.cuh"
#include "attn_backward.cuh"
#include "attn_bwd_fused.cuh"
#include "gemm_tcgen05.cuh"
#include "ln_backward.cuh"
#include "reduce_ln.cuh"
#include "simt_f32.cuh"
#include "tp_internal.h"

namespace {

using tp::MAX_SHARDS;
static_assert(MAX_SHARDS == TP_MAX_SHARDS, "shard limit mismatch");

constexpr int MAX_DEVICES = 64;

struct DeviceInfo {
  bool ready = false;
  bool ok = false;
  int sm_count = 0;
  int max_pairs = 0;  // co-resident CTA pairs of the cta_group::2 GEMM
};

// The reduce + residual + LayerNorm stages rows in shared memory with bulk
// copies (1) or loads them into registers (0).
#ifndef TP_RLN_BULK
#define TP_RLN_BULK 0
#endif

// The attention backward makes P and dS in one dual-accumulator GEMM (1) or in
// a score GEMM and a dP GEMM that reads P back (0).
// Attention backward: the fused key-major and query-major kernels (1), or
// per-head GEMM launches over P and dS in memory (0).
#ifndef TP_ATTN_BACK_FUSED
#define TP_ATTN_BACK_FUSED 1
#endif
#ifndef TP_ATTN_BACK_DUAL
#define TP_ATTN_BACK_DUAL 1
#endif

// Rows of 2049..4096 columns: 8 warps a row with 16 values a lane (0), or 16
// warps a row with 8 values a lane (1).
#ifndef TP_RLN_PF
#define TP_RLN_PF 1  // single-partial bf16 rows loaded one group ahead, on f32 pairs (reduce_residual_ln_pf2_kernel)
#endif
#ifndef TP_DB_N_FASTEST
#define TP_DB_N_FASTEST 1  // the MLP's dB GEMMs walk their tiles n fastest
#endif
#ifndef TP_RLN_4096_WPR
#define TP_RLN_4096_WPR 8  // warps per row of the reduce + LayerNorm kernel for 2048 < H <= 4096 (8 or 4)
#endif
#ifndef TP_RLN_WIDE_ROWS
#define TP_RLN_WIDE_ROWS 0
#endif

// Most K-split partial-sum slots a row-split GEMM feeding the LayerNorm may use.
#define TP_MAX_K_SPLITS 4

// GEMM flavour: CTA pairs (cta_group::2, 256-row tiles) unless the problem has
// at most 128 rows, where a pair would leave half of every tile empty.
#ifndef TP_GEMM_PAIR_MIN_ROWS
#define TP_GEMM_PAIR_MIN_ROWS 129
#endif

std::mutex g_mu;
DeviceInfo g_dev[MAX_DEVICES];
int g_force_tile_n = 0;  // tp_set_gemm_tile_n: 0 = cost model
int g_stream_k = 0;      // tp_set_gemm_stream_k: 0 = whole tiles, 1 = wherever a workspace allows, 2 = cost model
int g_attn_split = 1;    // tp_set_attn_kv_split: 0 = off, 1 = the last partial wave, 2 = every unit
unsigned long long g_sk_epoch = 0;  // last stream-K launch's epoch (see next_sk_epoch)
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// ------------------------------------------------------------ event timing
constexpr int PROF_CAP = 16384;  // launches timed between two collects
constexpr int PROF_KINDS = 8;
bool g_prof_on = false;
bool g_prof_sampling = true;  // record events for the launches made while set
bool g_prof_events_made = false;
cudaEvent_t g_ev_start[PROF_CAP];
cudaEvent_t g_ev_stop[PROF_CAP];
int g_prof_kind[PROF_CAP];
int g_prof_n = 0;
long long g_prof_launches[PROF_KINDS];  // every launch while enabled, timed or not

enum Kind {
  K_GEMM_TC = 0, K_REDUCE_LN = 1, K_GEMM_SIMT = 2, K_ATTN = 3, K_LN_BACK = 4, K_ATTN_BACK = 5, K_LN_PARAMS = 6,
  K_ATTN_BWD = 7
};

struct ProfScope {
  int slot = -1;
  cudaStream_t st;
  ProfScope(int kind, cudaStream_t s) : st(s) {
    if (!g_prof_on) return;
    ++g_prof_launches[kind];
    if (!g_prof_sampling || g_prof_n >= PROF_CAP) return;
    slot = g_prof_n++;
    g_prof_kind[slot] = kind;
    cudaEventRecord(g_ev_start[slot], st);
  }
  ~ProfScope() {
    if (slot >= 0) cudaEventRecord(g_ev_stop[slot], st);
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

template <int CG, bool WIDE, int FEAT>
bool gemm_smem_attr() {
  return cudaFuncSetAttribute(tp::gemm_tcgen05_kernel<CG, WIDE, FEAT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              tp::GemmCfg<CG, WIDE, FEAT>::SMEM_BYTES) == cudaSuccess;
}

// Resolve the current device's properties and the tensor-map encoder once.
int device_ready(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TP_ERR_NO_DEVICE;
  if (dev < 0 || dev >= MAX_DEVICES) return TP_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    d.ready = true;
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      d.ok = false;
    } else {
      d.ok = (major == 10);
      d.sm_count = sms;
    }
    if (d.ok) {
      if (!gemm_smem_attr<1, false, tp::FEAT_BASE>() || !gemm_smem_attr<2, false, tp::FEAT_BASE>() ||
          !gemm_smem_attr<2, true, tp::FEAT_BASE>() || !gemm_smem_attr<1, false, tp::FEAT_SK>() ||
          !gemm_smem_attr<2, false, tp::FEAT_SK>() || !gemm_smem_attr<2, true, tp::FEAT_SK>() ||
          !gemm_smem_attr<1, false, tp::FEAT_DUAL>() || !gemm_smem_attr<2, false, tp::FEAT_DUAL>() ||
          cudaFuncSetAttribute(tp::attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tp::attn::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(tp::attn_bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tp::attb::SMEM_DKV) != cudaSuccess ||
          cudaFuncSetAttribute(tp::attn_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tp::attb::SMEM_DQ) != cudaSuccess)
        d.ok = false;
    }
    if (d.ok) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
      cfg.blockDim = dim3(tp::GemmCfg<2>::NUM_THREADS, 1, 1);
      cfg.dynamicSmemBytes = tp::GemmCfg<2>::SMEM_BYTES;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int pairs = 0;
      if (cudaOccupancyMaxActiveClusters(&pairs, tp::gemm_tcgen05_kernel<2>, &cfg) != cudaSuccess || pairs < 1)
        d.ok = false;
      d.max_pairs = pairs;
    }
    if (d.ok && !g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        d.ok = false;
      else
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  if (!d.ok) return TP_ERR_NO_DEVICE;
  *out = &d;
  return TP_OK;
}

// 2-D bf16 tensor map over a row-major matrix [rows, cols] with a row stride of
// `ld` elements; box {box_cols, box_rows}; 128-byte swizzle; OOB reads give 0.
bool tmap_bf16(CUtensorMap* m, const void* base, long long rows, long long cols, long long ld, int box_cols,
               int box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2u};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D output map {cols, rows, slots} over row-major [slots][rows][ld] (f32 or
// bf16); box {128 bytes of columns, 128 rows (32 with per-warp epilogue
// stores), 1 slot}; 128-byte swizzle.  TMA stores through it write nothing
// outside [cols] x [rows] x [slots].
bool tmap_out(CUtensorMap* m, void* base, int f32, long long cols, long long rows, long long slots, long long ld,
              long long slot_stride) {
  const cuuint64_t es = f32 ? 4u : 2u;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(slots)};
  const long long ss = slot_stride > 0 ? slot_stride : rows * ld;
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * es, static_cast<cuuint64_t>(ss) * es};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / es), TP_GEMM_WARP_STORES ? 32u : 128u, 1u};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA; }

// Launch with programmatic stream serialization: the kernel may be scheduled
// before the preceding kernel in the stream ends and waits for it itself
// (griddep_wait) before touching data that kernel produced.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Tile plan of a tensor-core GEMM: tile width (256, or 288..512 for wide
// tiles) and number of K splits, from a small cost model of a persistent
// launch on `slots` SM pairs, calibrated by timing these kernels on B200
// under its power cap:
//  * Main loop: waves x k-blocks per unit x the time of one k-block, about
//    0.40 us for a 256 x 256 x 64 pair step.  A w-column tile does w/256 of
//    that MMA work, at a lower time per MAC because every operand byte feeds
//    more MACs (the main loop is bound by operand traffic from L2): relative
//    time per MAC 1.0 at w = 256, 0.95 at 384, 0.88 at 448, 0.82 at 480 and
//    0.75 at 512 (linear in between).  The 512 figure is the sustained one:
//    0.78 on a cool GPU, but moving fewer operand bytes per MAC also draws
//    less power, and under the power cap the clock stays higher (the MLP
//    sublayer step at S2048 H4096 F16384 ran 2.1 % faster over 2000 steps
//    with both GEMMs at 512 than with 256 and 480).
//  * Every extra f32 partial slot of a K split costs one write and one read of
//    M x N x 4 bytes at HBM speed (the reduce + LayerNorm kernel adds slots).
//  * A wide tile fills TMEM, so its epilogue no longer overlaps the next
//    tile's main loop: each wave but the last pays it (about 3.5 us per 256
//    columns, twice that for an epilogue that also stores the pre-activation
//    or reads a second operand: U, P).
struct TilePlan {
  int tile_n = 256;
  int splits = 1;
  int stream_k = 0;   // 1: stream-K over `sk_clusters` clusters
  int sk_clusters = 0;
};

// Workspace a stream-K launch needs: a 128 x w f32 partial block per CTA of
// each of `clusters` clusters of cg CTAs, then one 8-byte flag per CTA.
// A stream-K split is usable when no remainder tile's tail has more producer
// pieces than a finisher lists (tp::SK_MAX_PRODUCERS).
bool sk_split_ok(long long tiles, int kbt, int clusters) {
  const tp::SkSplit sp = tp::sk_split(tiles, kbt, clusters);
  if (sp.m == 0) return false;
  int list[tp::SK_MAX_PRODUCERS + 1];
  for (int r = 0; r < sp.R; ++r)
    if (tp::sk_producers(sp, kbt, clusters, r, list, tp::SK_MAX_PRODUCERS + 1) > tp::SK_MAX_PRODUCERS) return false;
  return true;
}

size_t sk_bytes(long long clusters, int cg, int w) {
  return align256(static_cast<size_t>(clusters) * cg * 128 * w * 4) + static_cast<size_t>(clusters) * cg * 8;
}

// Flags of stream-K launches carry the launch's epoch, so a flag left by an
// earlier launch never matches.  The epochs start from a process-specific
// salt in the high half, so stale workspace contents from another process
// are not mistaken for this one's either.
unsigned long long next_sk_epoch() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sk_epoch == 0) {
    const unsigned long long salt =
        (static_cast<unsigned long long>(reinterpret_cast<uintptr_t>(&g_sk_epoch)) >> 4) ^
        static_cast<unsigned long long>(std::chrono::steady_clock::now().time_since_epoch().count());
    g_sk_epoch = (salt | 1ull) << 32;
  }
  return ++g_sk_epoch;
}

constexpr double T_KB = 0.40e-6;
constexpr double T_EPI_256 = 3.5e-6;
// An M-major A (the weight-gradient GEMMs: X^T, G^T, O^T) costs the
// 256-column tiles 10 % more per k-block than the model's K-major figure,
// relative to the wide tiles: measured (ncu, one box) dWqkv 692.6 against
// 634.5 us, dWo 238.2 against 222.1, the MLP's dA 243.1 against 221.9 and
// dB 243.3 against 222.4 us at 256 and 512 columns.
constexpr double MN_A_PENALTY_256 = 1.10;

double per_mac_factor(int w) {
  static const int xs[] = {256, 384, 448, 480, 512};
  static const double ys[] = {1.0, 0.95, 0.88, 0.82, 0.75};
  if (w <= xs[0]) return ys[0];
  for (int i = 1; i < 5; ++i)
    if (w <= xs[i]) return ys[i - 1] + (ys[i] - ys[i - 1]) * (w - xs[i - 1]) / double(xs[i] - xs[i - 1]);
  return ys[4];
}

double kb_cost(int w) { return (w / 256.0) * per_mac_factor(w); }

long long n_blocks_for(const tp::GemmArgs& p, int w) {
  const long long per_shard = (p.shard_n + w - 1) / w;
  return p.row_mode ? per_shard : per_shard * p.t;
}

// The data-parallel plan: whole tiles dealt round-robin to the clusters,
// optionally with the K loop split into f32 slots.
TilePlan plan_tiles_dp(const tp::GemmArgs& p, bool pair, int slots, int max_splits, double* cost) {
  TilePlan best;
  const long long m_blocks = (p.M + (pair ? 255 : 127)) / (pair ? 256 : 128);
  const long long out_elems = static_cast<long long>(p.M) * (p.row_mode ? p.shard_n : p.shard_n * p.t);
  const double slot_cost = static_cast<double>(out_elems) * 8.0 / 6.0e12;
  const long long tiles = m_blocks * n_blocks_for(p, 256);
  double best_t = 1e30;
  for (int s = 1; s <= max_splits && s <= p.k_blocks; ++s) {
    const long long waves = (tiles * s + slots - 1) / slots;
    const long long kb = (p.k_blocks + s - 1) / s;
    const double t = static_cast<double>(waves * kb) * T_KB * (p.a_mnmajor ? MN_A_PENALTY_256 : 1.0) +
                     (s - 1) * slot_cost;
    if (t < best_t * 0.98) {  // a split must buy at least 2%
      best_t = t;
      best.splits = s;
    }
  }
  const int step = p.out_f32 ? 32 : 64;  // a 128-byte output chunk must not cross a tile edge
  *cost = best_t;
  if (g_force_tile_n) {
    best.splits = 1;
    if (g_force_tile_n == 128) {  // narrow tiles, single CTAs included
      best.tile_n = 128;
      return best;
    }
    if (!pair) return best;
    best.tile_n = (g_force_tile_n + step - 1) / step * step;
    if (best.tile_n > 512) best.tile_n = 512;
    return best;
  }
  // Shards of at most 128 columns with an N-major B: 128-column tiles, whose
  // N = 128 MMA does no work on columns past the shard (same tile count).
  if (p.shard_n <= 128 && !p.b_kmajor) {
    best.tile_n = 128;
    return best;
  }
  if (!pair) return best;
  const double epi_weight = p.epi_mode == tp::EPI_PLAIN ? 1.0 : 2.0;
  for (int w = 256 + step; w <= 512; w += step) {
    const long long wt = m_blocks * n_blocks_for(p, w);
    const long long waves = (wt + slots - 1) / slots;
    const double t = static_cast<double>(waves * p.k_blocks) * kb_cost(w) * T_KB +
                     static_cast<double>(waves - 1) * (w / 256.0) * T_EPI_256 * epi_weight;
    if (t < best_t * 0.98) {  // wide tiles must buy at least 2%
      best_t = t;
      best.tile_n = w;
      best.splits = 1;
    }
  }
  *cost = best_t;
  return best;
}

// Stream-K (tp::sk_split): the whole waves as in the data-parallel plan, then
// the remainder tiles split along K between their head clusters and the spare
// clusters, so the last wave takes about R kbt / P k-blocks instead of kbt.
// Plus the exposed epilogue of every piece but the last with wide tiles, plus
// the fixed cost of the split tiles' partials (the producers' stores, the
// finishers' wait and reads: about 3 us).
constexpr double T_SK_FIX = 3.0e-6;

double sk_cost(const tp::GemmArgs& p, bool pair, int clusters, int w) {
  const long long m_blocks = (p.M + (pair ? 255 : 127)) / (pair ? 256 : 128);
  const long long tiles = m_blocks * n_blocks_for(p, w);
  const tp::SkSplit sp = tp::sk_split(tiles, p.k_blocks, clusters);
  const long long last = sp.R == 0 ? 0 : (sp.m == 0 ? p.k_blocks : sp.m);
  const long long steps = static_cast<long long>(sp.W) * p.k_blocks + last;
  const double epi_weight = p.epi_mode == tp::EPI_PLAIN ? 1.0 : 2.0;
  const long long exposed = w > 256 ? sp.W : 0;
  return static_cast<double>(steps) * kb_cost(w) * T_KB + T_SK_FIX +
         static_cast<double>(exposed) * (w / 256.0) * T_EPI_256 * epi_weight;
}

// The tile plan: the data-parallel one, or stream-K where the caller gives a
// workspace of `sk_area` bytes for the partials (0: none), the epilogue is the
// plain one, and it is at least 2 % faster by the cost model.
TilePlan plan_tiles(const tp::GemmArgs& p, bool pair, int slots, int max_splits, size_t sk_area = 0) {
  double best_t = 0.0;
  TilePlan best = plan_tiles_dp(p, pair, slots, max_splits, &best_t);
  if (g_stream_k == 0 || sk_area == 0 || p.epi_mode != tp::EPI_PLAIN) return best;
  const int cg = pair ? 2 : 1;
  const int step = p.out_f32 ? 32 : 64;
  const long long m_blocks = (p.M + (pair ? 255 : 127)) / (pair ? 256 : 128);
  if (g_stream_k == 1) {
    // Forced (tests): the data-parallel plan's width (or the forced width),
    // over as many clusters as the workspace holds partial blocks for.
    long long clusters = slots;
    while (clusters >= 2 && sk_bytes(clusters, cg, best.tile_n) > sk_area) --clusters;
    const long long steps = m_blocks * n_blocks_for(p, best.tile_n) * p.k_blocks;
    if (clusters >= 2 && steps >= clusters &&
        sk_split_ok(m_blocks * n_blocks_for(p, best.tile_n), p.k_blocks, static_cast<int>(clusters))) {
      best.stream_k = 1;
      best.sk_clusters = static_cast<int>(clusters);
      best.splits = 1;
    }
    return best;
  }
  if (g_force_tile_n || best.tile_n == 128) return best;  // a forced width, or narrow shards: as planned
  for (int w = 256; w <= (pair ? 512 : 256); w += step) {
    if (sk_bytes(slots, cg, w) > sk_area) continue;
    if (!sk_split_ok(m_blocks * n_blocks_for(p, w), p.k_blocks, slots)) continue;  // nothing (usable) to split
    const double t = sk_cost(p, pair, slots, w);
    if (t < best_t * 0.98) {
      best_t = t;
      best.tile_n = w;
      best.splits = 1;
      best.stream_k = 1;
      best.sk_clusters = slots;
    }
  }
  return best;
}

// Options of a tensor-core GEMM beyond the forward sublayers' needs (the
// backward pass): M-major A, strided B shards, per-shard output buffers, and
// the epilogue modes of tp::GemmArgs.
struct GemmExtra {
  int a_mnmajor = 0;                 // A stored [K, M] (row stride lda)
  int n_fastest = 0;                 // tiles walk n fastest (GemmArgs::n_fastest)
  long long ldb = 0;                 // row stride of every B shard (0: contiguous)
  void* const* C_shards = nullptr;   // column mode: shard s writes C_shards[s] (row stride ldc_shard)
  long long ldc_shard = 0;
  int epi_mode = tp::EPI_PLAIN;
  const void* aux = nullptr;         // EPI_AUX_PRE: bf16 output laid out like C; EPI_GRAD: bf16 U
  long long ld_aux = 0;
  int m_split = 0;                   // column mode, t = 1: output rows split into m_split buffers
                                     // C_shards[s] of M / m_split rows each (a multiple of 256)
  const void* const* A_shards = nullptr;  // column mode: shard s reads its own A_shards[s] (same
                                          // shape and lda as A): t independent products in one launch
  const float* rowvec = nullptr;     // EPI_SOFTMAX / EPI_DSOFTMAX: row values r, shard s at
  long long rowvec_ld = 0;           //   rowvec + s * rowvec_ld
  float epi_scale = 1.0f;
  void* sk_ws = nullptr;             // scratch the launch may use for stream-K partials and flags
  size_t sk_ws_bytes = 0;            //   (256-byte aligned; 0: no stream-K)
  // Dual accumulators (column mode, K-major B, EPI_DUAL_SOFTMAX): a second
  // product A2_s B2_s of the same shape per shard, its A with row stride lda2
  // and its B with row stride ldb2; the second output (dS) goes to `aux`.
  const void* const* A2_shards = nullptr;
  long long lda2 = 0;
  const void* const* B2_shards = nullptr;
  long long ldb2 = 0;
  const float* rowvec2 = nullptr;
  float epi_scale2 = 1.0f;
};

template <int CG, bool WIDE, int FEAT>
int launch_gemm_tc(const DeviceInfo& dev, tp::GemmArgs& p, const TilePlan& plan, const GemmExtra& ex,
                   cudaStream_t st) {
  using C = tp::GemmCfg<CG, WIDE, FEAT>;
  p.m_blocks = ceil_div(p.M, C::TILE_M);
  p.tile_n = plan.tile_n;
  p.n2 = WIDE ? plan.tile_n - C::BN : 0;
  p.idesc2 = WIDE ? tp::idesc_bf16_f32(C::TILE_M, p.n2, p.a_mnmajor != 0, !p.b_kmajor) : 0u;
  p.n_blocks_per_shard = ceil_div(p.shard_n, p.tile_n);
  p.n_blocks = p.row_mode ? p.n_blocks_per_shard : p.n_blocks_per_shard * p.t;
  const long long tiles = static_cast<long long>(p.m_blocks) * p.n_blocks;
  const int slots = CG == 2 ? dev.max_pairs : dev.sm_count;
  p.splits = plan.splits;
  const long long es = p.out_f32 ? 4 : 2;
  if (ex.m_split > 0) {
    p.m_split_rows = p.M / ex.m_split;
    for (int s = 0; s < ex.m_split; ++s)
      if (!tmap_out(&p.tmC[s], ex.C_shards[s], p.out_f32, p.shard_n, p.m_split_rows, 1, ex.ldc_shard, 0))
        return TP_ERR_CUDA;
  } else if (p.row_mode) {
    if (!tmap_out(&p.tmC[0], p.C, p.out_f32, p.shard_n, p.M, p.splits, p.ldc, p.slot_stride)) return TP_ERR_CUDA;
  } else {
    for (int s = 0; s < p.t; ++s) {
      void* base = ex.C_shards ? ex.C_shards[s] : static_cast<uint8_t*>(p.C) + static_cast<long long>(s) * p.shard_n * es;
      const long long ld = ex.C_shards ? ex.ldc_shard : p.ldc;
      if (!tmap_out(&p.tmC[s], base, p.out_f32, p.shard_n, p.M, 1, ld, 0)) return TP_ERR_CUDA;
      if (ex.epi_mode == tp::EPI_AUX_PRE || ex.epi_mode == tp::EPI_DUAL_SOFTMAX) {
        void* abase = static_cast<uint8_t*>(const_cast<void*>(ex.aux)) + static_cast<long long>(s) * p.shard_n * 2;
        if (!tmap_out(&p.tmAux[s], abase, 0, p.shard_n, p.M, 1, ex.ld_aux, 0)) return TP_ERR_CUDA;
      }
    }
  }
  const long long units = tiles * p.splits;
  int clusters = static_cast<int>(units < slots ? units : slots);
  if (FEAT == tp::FEAT_SK) {
    clusters = plan.sk_clusters;
    p.sk = 1;
    p.splits = 1;
    p.sk_ws = static_cast<float*>(ex.sk_ws);
    p.sk_flags = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(ex.sk_ws) +
                                                       align256(static_cast<size_t>(clusters) * CG * 128 * p.tile_n * 4));
    p.sk_epoch = next_sk_epoch();
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see griddep_wait in the kernel
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = CG;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.gridDim = dim3(clusters * CG, 1, 1);
  cfg.blockDim = dim3(C::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = CG == 2 ? 2 : 1;
  ProfScope ps(K_GEMM_TC, st);
  if (cudaLaunchKernelEx(&cfg, tp::gemm_tcgen05_kernel<CG, WIDE, FEAT>, p) != cudaSuccess) return TP_ERR_CUDA;
  return launch_status();
}

// Tensor-core GEMM.  Column mode: B shard s is [K, shard_n], output columns
// [s*shard_n, (s+1)*shard_n).  Row mode: B shard s is [shard_k, shard_n] and
// multiplies A's columns [s*shard_k, (s+1)*shard_k); all shards are summed.
// With b_kmajor every shard is stored transposed ([shard_n, shard_k], the
// nn.Linear [out, in] layout) and read K-major.
// With max_splits > 1 (f32 output only) the K loop may be cut into up to
// max_splits ranges whose partial sums land in slots `slot_stride` elements
// apart; *splits_out tells the caller how many slots to add.
int run_gemm_tc(const DeviceInfo& dev, const void* A, long long lda, int M, const void* const* B, int t,
                int row_mode, int shard_k, int shard_n, void* C, long long ldc, int out_f32, int act,
                cudaStream_t st, int max_splits = 1, long long slot_stride = 0, int* splits_out = nullptr,
                int b_kmajor = 0, const GemmExtra* extra = nullptr) {
  const GemmExtra none;
  const GemmExtra& ex = extra ? *extra : none;
  using G = tp::GemmCfg<1>;
  if (splits_out) *splits_out = 1;
  if (M == 0) return TP_OK;
  const bool pair = M >= TP_GEMM_PAIR_MIN_ROWS;
  tp::GemmArgs p;
  std::memset(&p, 0, sizeof(p));
  const long long K_total = row_mode ? static_cast<long long>(shard_k) * t : shard_k;
  if (ex.A_shards && (row_mode || ex.m_split > 0)) return TP_ERR_INVALID_ARG;
  const int na = ex.A_shards ? t : 1;
  for (int s = 0; s < na; ++s) {
    const void* a = ex.A_shards ? ex.A_shards[s] : A;
    if (ex.a_mnmajor) {  // stored [K, M]; box 64 m x 64 k
      if (!tmap_bf16(&p.tmA[s], a, K_total, M, lda, 64, G::BK)) return TP_ERR_CUDA;
    } else if (!tmap_bf16(&p.tmA[s], a, M, K_total, lda, G::BK, G::BM)) {
      return TP_ERR_CUDA;
    }
  }
  p.a_per_shard = ex.A_shards ? 1 : 0;
  for (int s = 0; s < t; ++s) {
    bool ok;
    if (b_kmajor)  // shard [shard_n rows, shard_k cols]; box 64 k x (BN / CG) rows
      ok = tmap_bf16(&p.tmB[s], B[s], shard_n, shard_k, ex.ldb ? ex.ldb : shard_k, G::BK,
                     pair ? tp::GemmCfg<2>::B_COLS_CTA : G::BN);
    else           // shard [shard_k rows, shard_n cols]; box 64 n x 64 k
      ok = tmap_bf16(&p.tmB[s], B[s], shard_k, shard_n, ex.ldb ? ex.ldb : shard_n, G::B_BOX_N, G::BK);
    if (!ok) return TP_ERR_CUDA;
  }
  const bool softmax_epi = ex.epi_mode == tp::EPI_SOFTMAX || ex.epi_mode == tp::EPI_DSOFTMAX ||
                           ex.epi_mode == tp::EPI_DUAL_SOFTMAX;
  if (softmax_epi && (out_f32 || row_mode || !ex.rowvec || (ex.epi_mode == tp::EPI_DSOFTMAX && !ex.aux)))
    return TP_ERR_INVALID_ARG;
  const bool dual = ex.epi_mode == tp::EPI_DUAL_SOFTMAX;
  if (dual) {
    // Dual accumulators: the second product's maps, shaped like the first's.
    if (!ex.A2_shards || !ex.B2_shards || !ex.rowvec2 || !ex.aux || !b_kmajor || ex.a_mnmajor || ex.m_split)
      return TP_ERR_INVALID_ARG;
    for (int s = 0; s < t; ++s) {
      if (!tmap_bf16(&p.tmA2[s], ex.A2_shards[s], M, K_total, ex.lda2, G::BK, G::BM) ||
          !tmap_bf16(&p.tmB2[s], ex.B2_shards[s], shard_n, shard_k, ex.ldb2, G::BK,
                     pair ? tp::GemmCfg<2>::B_COLS_CTA : G::BN))
        return TP_ERR_CUDA;
    }
    p.dual = 1;
    p.rowvec2 = ex.rowvec2;
    p.epi_scale2 = ex.epi_scale2;
  }
  p.a_mnmajor = ex.a_mnmajor;
  p.n_fastest = ex.n_fastest;
  p.epi_mode = ex.epi_mode;
  p.rowvec = ex.rowvec;
  p.rowvec_ld = ex.rowvec_ld;
  p.epi_scale = ex.epi_scale;
  p.aux = ex.aux;
  p.ld_aux = ex.ld_aux;
  p.C = C;
  p.ldc = ldc;
  p.M = M;
  p.t = t;
  p.row_mode = row_mode;
  p.shard_n = shard_n;
  p.shard_k = shard_k;
  p.N = row_mode ? shard_n : shard_n * t;
  p.k_blocks_per_shard = ceil_div(shard_k, G::BK);
  p.k_blocks = row_mode ? p.k_blocks_per_shard * t : p.k_blocks_per_shard;
  if (dual) p.k_blocks *= 2;  // the second product's k-blocks follow the first's
  p.act = act;
  p.out_f32 = out_f32;
  p.splits = 1;
  p.slot_stride = slot_stride;
  p.b_kmajor = b_kmajor;
  if (!out_f32) max_splits = 1;
  TilePlan plan = plan_tiles(p, pair, pair ? dev.max_pairs : dev.sm_count, max_splits,
                             (ex.sk_ws && ex.m_split == 0) ? ex.sk_ws_bytes : 0);
  if (dual) {  // both accumulators fill TMEM: 256-column tiles, one tile at a time
    plan = TilePlan();
    plan.tile_n = 256;
  }
  int r;
  if (dual) {
    r = pair ? launch_gemm_tc<2, false, tp::FEAT_DUAL>(dev, p, plan, ex, st)
             : launch_gemm_tc<1, false, tp::FEAT_DUAL>(dev, p, plan, ex, st);
  } else if (plan.stream_k) {
    if (!pair) r = launch_gemm_tc<1, false, tp::FEAT_SK>(dev, p, plan, ex, st);
    else if (plan.tile_n > tp::GemmCfg<2>::BN) r = launch_gemm_tc<2, true, tp::FEAT_SK>(dev, p, plan, ex, st);
    else r = launch_gemm_tc<2, false, tp::FEAT_SK>(dev, p, plan, ex, st);
  } else {
    if (!pair) r = launch_gemm_tc<1, false, tp::FEAT_BASE>(dev, p, plan, ex, st);
    else if (plan.tile_n > tp::GemmCfg<2>::BN) r = launch_gemm_tc<2, true, tp::FEAT_BASE>(dev, p, plan, ex, st);
    else r = launch_gemm_tc<2, false, tp::FEAT_BASE>(dev, p, plan, ex, st);
  }
  if (splits_out) *splits_out = p.splits;
  return r;
}

// f32 CUDA-core GEMM (same shard modes as run_gemm_tc).  With max_splits > 1
// (row mode, no activation) the K range may be cut over up to max_splits
// CTAs per tile, split z writing slot z at C + z * slot_stride; *splits_out
// tells the caller how many slots to add.
int run_gemm_simt(const float* A, long long lda, int M, const void* const* B, int t, int row_mode, int shard_k,
                  int shard_n, float* C, long long ldc, int act, cudaStream_t st, int b_kmajor = 0, int dev_sms = 148,
                  int max_splits = 1, long long slot_stride = 0, int* splits_out = nullptr) {
  if (splits_out) *splits_out = 1;
  if (M == 0) return TP_OK;
  tp::SimtArgs p;
  std::memset(&p, 0, sizeof(p));
  p.A = A;
  p.lda = lda;
  for (int s = 0; s < t; ++s) p.B[s] = static_cast<const float*>(B[s]);
  p.C = C;
  p.ldc = ldc;
  p.slot_stride = slot_stride;
  p.M = M;
  p.row_mode = row_mode;
  p.shard_n = shard_n;
  p.shard_k = shard_k;
  p.N = row_mode ? shard_n : shard_n * t;
  p.K = row_mode ? shard_k * t : shard_k;
  p.act = act;
  p.b_kmajor = b_kmajor;
  // Enough CTAs for two per SM where the K range allows it (each split keeps
  // at least two K chunks).
  const long long tiles = static_cast<long long>(ceil_div(p.N, tp::simt::TN)) * ceil_div(M, tp::simt::TM);
  const int chunks = ceil_div(p.K, tp::simt::TK);
  int splits = 1;
  if (act == TP_ACT_NONE && max_splits > 1) {
    while (splits < max_splits && tiles * splits < 2LL * dev_sms && chunks / (splits + 1) >= 2) ++splits;
  }
  p.splits = splits;
  if (splits_out) *splits_out = splits;
  dim3 grid(ceil_div(p.N, tp::simt::TN), ceil_div(M, tp::simt::TM), splits);
  ProfScope ps(K_GEMM_SIMT, st);
  tp::simt_gemm_f32_kernel<<<grid, tp::simt::THREADS, 0, st>>>(p);
  return launch_status();
}

// Y = LN(X + sum of the partials) (or the residual add alone).  The partials
// are `nparts` contiguous [S, H] slots starting at `parts`, or (parts == NULL)
// the list part_list[0..nparts); `ny_extra` further outputs y_extra[] receive
// the same values as Y.
int run_reduce_ln(int S, int H, int nparts, const float* parts, const void* X, int x_bf16, const float* gamma,
                  const float* beta, float eps, void* Y, int y_bf16, cudaStream_t st, int dev_sms,
                  int apply_ln = 1, const float* const* part_list = nullptr, int ny_extra = 0,
                  void* const* y_extra = nullptr, float* stats = nullptr) {
  if (S == 0) return TP_OK;
  tp::ReduceLnArgs p;
  std::memset(&p, 0, sizeof(p));
  p.apply_ln = apply_ln;
  p.stats = stats;
  p.S = S;
  p.H = H;
  p.nparts = nparts;
  p.parts = parts;
  p.part_stride = static_cast<long long>(S) * H;
  if (!parts && part_list) {
    for (int q = 0; q < nparts; ++q) p.part_ptr[q] = part_list[q];
    if (nparts == 1) p.parts = part_list[0];  // the single-partial kernel reads `parts`
  }
  p.ny_extra = ny_extra;
  for (int o = 0; o < ny_extra; ++o) p.y_extra[o] = y_extra[o];
  p.X = X;
  p.x_bf16 = x_bf16;
  p.gamma = gamma;
  p.beta = beta;
  p.eps = eps;
  p.Y = Y;
  p.y_bf16 = y_bf16;
  bool launched = true;
  ProfScope ps(K_REDUCE_LN, st);
#if TP_RLN_BULK
  // Rows staged in shared memory by bulk copies, `nst` rows ahead per CTA:
  // stages of up to 48 KiB are sized for two CTAs per SM (4 stages at most),
  // larger ones for one; rows too wide for two stages take the register
  // kernel below.
  {
    const size_t xb = x_bf16 ? 2 : 4;
    const size_t stage = ((static_cast<size_t>(H) * (xb + 4 * nparts)) + 127) & ~size_t(127);
    if (2 * stage <= static_cast<size_t>(tp::rlb::MAX_STAGE_SMEM)) {
      const size_t budget = stage <= 48 * 1024 ? 96 * 1024 : tp::rlb::MAX_STAGE_SMEM;
      int nst = static_cast<int>(budget / stage);
      nst = nst < 2 ? 2 : (nst > 4 ? 4 : nst);
      const size_t smem = static_cast<size_t>(nst) * stage;
      auto go_bulk = [&](auto kern) {
        int per_sm = 1;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
                cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, tp::rlb::THREADS, smem) != cudaSuccess ||
            per_sm < 1)
          per_sm = 1;
        const int grid = S < per_sm * dev_sms ? S : per_sm * dev_sms;
        if (launch_pdl(kern, dim3(grid), dim3(tp::rlb::THREADS), smem, st, p, nst, static_cast<int>(stage)) !=
            cudaSuccess)
          launched = false;
      };
      const int ch = (H + 2047) / 2048;
      using namespace tp;
      switch (ch) {
        case 1: go_bulk(reduce_residual_ln_bulk_kernel<1>); break;
        case 2: go_bulk(reduce_residual_ln_bulk_kernel<2>); break;
        case 3: go_bulk(reduce_residual_ln_bulk_kernel<3>); break;
        case 4: go_bulk(reduce_residual_ln_bulk_kernel<4>); break;
        case 5: case 6: go_bulk(reduce_residual_ln_bulk_kernel<6>); break;
        default: go_bulk(reduce_residual_ln_bulk_kernel<8>); break;
      }
      const int ls = launch_status();
      return launched ? ls : TP_ERR_CUDA;
    }
  }
#endif
  // WPR warps per row (each lane holds CH chunks of 8 values); max(1, 8 / WPR)
  // rows per CTA; a grid of the resident CTA count walks the row groups.
  const bool np1 = nparts == 1;
  auto go = [&](auto kern, int wpr, int rows_per_cta) {
    const int threads = tp::rln::cta_threads(wpr);
    const int groups = ceil_div(S, rows_per_cta);
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0) != cudaSuccess || per_sm < 1)
      per_sm = 1;
    const int grid = groups < per_sm * dev_sms ? groups : per_sm * dev_sms;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see griddep_wait in the kernel
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) launched = false;
  };
  using namespace tp;
  if (H <= 512) np1 ? go(reduce_residual_ln_kernel<1, 2, true>, 1, 8) : go(reduce_residual_ln_kernel<1, 2, false>, 1, 8);
  else if (H <= 1024) np1 ? go(reduce_residual_ln_kernel<2, 2, true>, 2, 4) : go(reduce_residual_ln_kernel<2, 2, false>, 2, 4);
  else if (H <= 2048) np1 ? go(reduce_residual_ln_kernel<4, 2, true>, 4, 2) : go(reduce_residual_ln_kernel<4, 2, false>, 4, 2);
#if TP_RLN_WIDE_ROWS
  // one 512-thread CTA per row, 8 values per lane: fewer registers, more CTAs per SM
  else if (H <= 4096) np1 ? go(reduce_residual_ln_kernel<16, 1, true>, 16, 1) : go(reduce_residual_ln_kernel<16, 1, false>, 16, 1);
#elif TP_RLN_4096_WPR == 4
  // two rows per 256-thread CTA, 4 warps and 4 chunks per lane each
  else if (H <= 4096 && TP_RLN_PF && np1 && x_bf16 && apply_ln) go(reduce_residual_ln_pf2_kernel<4, 4>, 4, 2);
  else if (H <= 4096) np1 ? go(reduce_residual_ln_kernel<4, 4, true>, 4, 2) : go(reduce_residual_ln_kernel<4, 4, false>, 4, 2);
#else
  else if (H <= 4096 && TP_RLN_PF && np1 && x_bf16 && apply_ln) go(reduce_residual_ln_pf2_kernel<8, 2>, 8, 1);
  else if (H <= 4096) np1 ? go(reduce_residual_ln_kernel<8, 2, true>, 8, 1) : go(reduce_residual_ln_kernel<8, 2, false>, 8, 1);
#endif
  else if (H <= 8192 && TP_RLN_PF && np1 && x_bf16 && apply_ln) go(reduce_residual_ln_pf2_kernel<8, 4>, 8, 1);
  else if (H <= 8192) np1 ? go(reduce_residual_ln_kernel<8, 4, true>, 8, 1) : go(reduce_residual_ln_kernel<8, 4, false>, 8, 1);
  // (one-row CTAs of 12 or 16 warps keep the generic loop: fewer registers, two CTAs per SM)
  else if (H <= 12288) go(reduce_residual_ln_kernel<12, 4, false>, 12, 1);
  else go(reduce_residual_ln_kernel<16, 4, false>, 16, 1);
  const int ls = launch_status();
  return launched ? ls : TP_ERR_CUDA;
}

bool valid_dtype(int d) { return d == TP_DTYPE_F32 || d == TP_DTYPE_BF16; }
bool valid_act(int a) { return a >= TP_ACT_NONE && a <= TP_ACT_RELU; }
bool valid_out(int dtype, int out) {
  if (!valid_dtype(dtype) || !valid_dtype(out)) return false;
  return dtype == TP_DTYPE_BF16 || out == TP_DTYPE_F32;
}
bool shards_ok(const void* const* s, int t) {
  if (!s) return false;
  for (int i = 0; i < t; ++i)
    if (!s[i] || !aligned16(s[i])) return false;
  return true;
}
bool ptr_ok(const void* p) { return p && aligned16(p); }
bool opt_ptr_ok(const void* p) { return !p || aligned16(p); }
bool hidden_ok(int H) { return H >= 8 && H % 8 == 0 && H <= tp::rln::MAX_H; }

// ------------------------------------------------------------ training state
// Saved by tp_mlp_forward_train for tp_mlp_backward: U = X A (pre-activation,
// bf16 [S, F]), G = Act(U) (bf16 [S, F], the row-split GEMM's input),
// V = G B (f32 [S, H], the row-split GEMM's output before the residual) and
// the LayerNorm's row statistics (mean, 1/sqrt(var + eps); f32 [S][2]).
struct TrainState {
  size_t off_u, off_g, off_v, off_stats, bytes;
};
TrainState train_state_layout(int S, int H, int F) {
  TrainState t;
  const size_t sf = static_cast<size_t>(S) * F, sh = static_cast<size_t>(S) * H;
  t.off_u = 0;
  t.off_g = align256(sf * 2);
  t.off_v = t.off_g + align256(sf * 2);
  t.off_stats = t.off_v + align256(sh * 4);
  t.bytes = t.off_stats + align256(static_cast<size_t>(S) * 8);
  return t;
}

// Backward workspace: dZ (bf16 [S, H]), dU (bf16 [S, F]), the f32 row-split
// partial of dX ([S, H]) and the LayerNorm-backward CTAs' dgamma/dbeta partial
// rows (at most LNB_MAX_CTAS x 2 x H f32).
constexpr int LNB_MAX_CTAS = 640;
struct BackWs {
  size_t off_dz, off_du, off_dxp, off_part, bytes;
};
BackWs back_ws_layout(int S, int H, int F) {
  BackWs w;
  const size_t sf = static_cast<size_t>(S) * F, sh = static_cast<size_t>(S) * H;
  w.off_dz = 0;
  w.off_du = align256(sh * 2);
  w.off_dxp = w.off_du + align256(sf * 2);
  w.off_part = w.off_dxp + align256(sh * 4);
  w.bytes = w.off_part + align256(static_cast<size_t>(LNB_MAX_CTAS) * 2 * H * 4);
  return w;
}

// LayerNorm backward + the dgamma/dbeta reduction.  256-thread CTAs, one row
// at a time each, CH = ceil(H / 2048) chunks of 8 per thread; as many CTAs as
// are resident (at most LNB_MAX_CTAS, at most S), each with 8 H bytes of
// shared memory for its per-column sums.  stats: the forward's row (mean, r).
int run_ln_backward(int S, int H, const float* V, const float* stats, const void* X, const void* dY,
                    const float* gamma, void* dZ, float* partial, float* dgamma, float* dbeta, cudaStream_t st,
                    int dev_sms) {
  tp::LnBackArgs p;
  p.S = S;
  p.H = H;
  p.V = V;
  p.stats = stats;
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.dY = static_cast<const __nv_bfloat16*>(dY);
  p.gamma = gamma;
  p.dZ = static_cast<__nv_bfloat16*>(dZ);
  p.partial = partial;
  const size_t smem = static_cast<size_t>(H) * 8;
  int grid = 0;
  cudaError_t le = cudaSuccess;
  auto go = [&](auto kern) {
    int per_sm = 1;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, tp::lnb::THREADS, smem) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    grid = per_sm * dev_sms;
    if (grid > LNB_MAX_CTAS) grid = LNB_MAX_CTAS;
    if (grid > S) grid = S;
    le = launch_pdl(kern, dim3(grid), dim3(tp::lnb::THREADS), smem, st, p);
  };
  {
    ProfScope ps(K_LN_BACK, st);
    switch ((H + 2047) / 2048) {
      case 1: go(tp::ln_backward_kernel<1>); break;
      case 2: go(tp::ln_backward_kernel<2>); break;
      case 3: case 4: go(tp::ln_backward_kernel<4>); break;
      default: go(tp::ln_backward_kernel<8>); break;
    }
    if (le != cudaSuccess || launch_status() != TP_OK) return TP_ERR_CUDA;
  }
  if (dgamma || dbeta) {
    ProfScope ps(K_LN_PARAMS, st);
    const cudaError_t pe = launch_pdl(tp::ln_grad_params_kernel, dim3(ceil_div(H, 32)),
                                      dim3(32 * tp::LNB_PARAM_SLICES), 0, st, static_cast<const float*>(partial),
                                      grid, H, dgamma, dbeta);
    return pe != cudaSuccess ? TP_ERR_CUDA : launch_status();
  }
  return TP_OK;
}

}  // namespace

extern "C" {

int tp_version(void) { return TP_API_VERSION; }

const char* tp_status_string(int s) {
  switch (s) {
    case TP_OK: return "ok";
    case TP_ERR_INVALID_ARG: return "invalid argument";
    case TP_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case TP_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case TP_ERR_CUDA: return "CUDA error";
    case TP_ERR_TIMEOUT: return "device-side wait timed out";
    case TP_ERR_NO_DEVICE: return "no sm_100 device";
    default: return "unknown status";
  }
}

int tp_device_error(void) {
  DeviceInfo* dev = nullptr;
  int st = device_ready(&dev);
  if (st != TP_OK) return st;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, tp::g_tp_device_error, sizeof(int)) != cudaSuccess) return TP_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(tp::g_tp_device_error, &zero, sizeof(int)) != cudaSuccess) return TP_ERR_CUDA;
  return v == 0 ? TP_OK : TP_ERR_TIMEOUT;
}

// ------------------------------------------------------------------- MLP
size_t tp_mlp_workspace_bytes(int S, int H, int F, int t, int dtype) {
  if (S < 0 || H <= 0 || F <= 0 || t < 1 || !valid_dtype(dtype)) return 0;
  (void)t;
  const size_t eh = dtype == TP_DTYPE_BF16 ? 2 : 4;
  return align256(static_cast<size_t>(S) * F * eh) + TP_MAX_K_SPLITS * static_cast<size_t>(S) * H * 4;
}

}  // extern "C"

namespace {

// The two products of the MLP sublayer on `in` ([S, H]): Hbuf = Act(in A_i) in
// the column slices of an [S, F] buffer, then Zsum = sum_i Hbuf_i B_i (f32
// [S, H]; the K loop may be cut into up to max_splits ranges, *nparts of them
// used, one slot of S*H floats each).  Arguments are already checked.
int mlp_products(const DeviceInfo& dev, int S, int H, int F, int t, int dtype, const void* in,
                 const void* const* A_shards, const void* const* B_shards, int act, void* Hbuf, float* Zsum,
                 int max_splits, int* nparts, cudaStream_t s, int kmaj, void* sk_ws = nullptr,
                 size_t sk_bytes = 0) {
  *nparts = 1;
  if (S == 0) return TP_OK;
  const int Fs = F / t;
  int st;
  if (dtype == TP_DTYPE_BF16) {
    GemmExtra ex;  // scratch for stream-K partials (its plan never also splits K into slots)
    ex.sk_ws = sk_ws;
    ex.sk_ws_bytes = sk_bytes;
    // H_i = Act(in A_i) into columns [i Fs, (i+1) Fs) of Hbuf [S, F] (bf16).
    st = run_gemm_tc(dev, in, H, S, A_shards, t, /*row_mode=*/0, /*shard_k=*/H, /*shard_n=*/Fs, Hbuf, F,
                     /*out_f32=*/0, act, s, 1, 0, nullptr, kmaj, &ex);
    if (st != TP_OK) return st;
    // Zsum = sum_i H_i B_i, accumulated in TMEM across the shards (f32).
    return run_gemm_tc(dev, Hbuf, F, S, B_shards, t, /*row_mode=*/1, /*shard_k=*/Fs, /*shard_n=*/H, Zsum, H,
                       /*out_f32=*/1, TP_ACT_NONE, s, max_splits, static_cast<long long>(S) * H, nparts, kmaj, &ex);
  }
  st = run_gemm_simt(static_cast<const float*>(in), H, S, A_shards, t, 0, H, Fs, static_cast<float*>(Hbuf), F, act,
                     s, kmaj, dev.sm_count);
  if (st != TP_OK) return st;
  return run_gemm_simt(static_cast<const float*>(Hbuf), F, S, B_shards, t, 1, Fs, H, Zsum, H, TP_ACT_NONE, s, kmaj,
                       dev.sm_count, max_splits, static_cast<long long>(S) * H, nparts);
}

// MLP sublayer on `in` with residual `res`: Y = LN(res + sum_i Act(in A_i) B_i),
// or Y = res + sum_i Act(in A_i) B_i without the LayerNorm (apply_ln = 0).
// Arguments are already checked.
int mlp_core(const DeviceInfo& dev, int S, int H, int F, int t, int dtype, int out_dtype, const void* in,
             const void* res, const void* const* A_shards, const void* const* B_shards, const float* gamma,
             const float* beta, float eps, int act, int apply_ln, void* Y, void* workspace, cudaStream_t s,
             int kmaj = 0) {
  if (S == 0) return TP_OK;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t eh = dtype == TP_DTYPE_BF16 ? 2 : 4;
  void* Hbuf = ws;
  float* Zsum = reinterpret_cast<float*>(ws + align256(static_cast<size_t>(S) * F * eh));
  int nparts = 1;
  // Slots 1.. of the partial-sum area double as stream-K scratch: a stream-K
  // plan writes slot 0 only.
  const size_t sh4 = static_cast<size_t>(S) * H * 4;
  int st = mlp_products(dev, S, H, F, t, dtype, in, A_shards, B_shards, act, Hbuf, Zsum, TP_MAX_K_SPLITS, &nparts, s,
                        kmaj, reinterpret_cast<uint8_t*>(Zsum) + sh4, (TP_MAX_K_SPLITS - 1) * sh4);
  if (st != TP_OK) return st;
  return run_reduce_ln(S, H, nparts, Zsum, res, dtype == TP_DTYPE_BF16, gamma, beta, eps, Y,
                       out_dtype == TP_DTYPE_BF16, s, dev.sm_count, apply_ln);
}

// Attention sublayer on `in` with residual `res` (bf16): Y = LN(res + O Wo)
// or Y = res + O Wo (apply_ln = 0).  Arguments are already checked.
// Kept by a training forward of the attention sublayer: the buffers it writes
// anyway (QKV, O, the O projection's f32 output) and each row's log2 softmax
// denominator per head.
struct AttnKeep {
  void* qkv = nullptr;
  void* o = nullptr;
  float* zsum = nullptr;
  float* lse2 = nullptr;
  float* stats = nullptr;  // the LayerNorm's row (mean, 1/sqrt(var + eps))
};

// QKV, per-head attention and the row-split O projection of the nh heads held
// by t shards (nh / t each) of a model of hidden size H: QKV [S, 3 nh d] and O
// [S, nh d] bf16 in the given buffers, Zsum = sum_s O_s Wo_s (f32 [S, H]; up to
// max_splits K-split slots, *nparts used).  Arguments are already checked.
// Last-wave key split of the attention kernel (see attention.cuh): of U =
// nh * ceil(S / 256) units on `slots` resident CTAs, the R = U mod slots of
// the last partial wave run as two half-key-range CTAs each when 2R CTAs fit
// in one wave (mode 1), or every unit does (mode 2, for tests).  Scratch:
// partial O rows, (m, l) rows and flags per split unit.
struct AttnSplit {
  int whole, split, kv_half;
};

size_t attn_split_bytes(long long R) {
  return align256(static_cast<size_t>(R) * 8 * 32 * tp::attn::D * 4) + align256(static_cast<size_t>(R) * 8 * 64 * 4) +
         static_cast<size_t>(R) * 8 * 2 * 8;
}

AttnSplit attn_split_plan(int S, int nh, int slots, int mode, size_t scratch_bytes) {
  const int per = tp::attn::TILES * tp::attn::BQ;
  const long long U = static_cast<long long>(nh) * ((S + per - 1) / per);
  const int nkv = S / tp::attn::BKV;
  AttnSplit p{static_cast<int>(U), 0, 0};
  if (mode == 0 || U == 0 || slots < 2 || nkv < 2) return p;
  long long R;
  if (mode == 2) {
    R = U;
  } else {
    if (nkv < 4) return p;  // halves of one key block gain nothing
    R = U % slots;
    if (R == 0 || 2 * R > slots) return p;
  }
  if (attn_split_bytes(R) > scratch_bytes) return p;
  p.whole = static_cast<int>(U - R);
  p.split = static_cast<int>(R);
  p.kv_half = nkv / 2;
  return p;
}

int attn_products(const DeviceInfo& dev, int S, int H, int nh, int d, int t, const void* in,
                  const void* const* Wqkv_shards, const void* const* Wo_shards, void* QKV, void* Obuf, float* Zsum,
                  int max_splits, int* nparts, cudaStream_t s, int kmaj, float* lse2, void* sk_ws = nullptr,
                  size_t sk_bytes = 0, size_t zsum_bytes = 0) {
  *nparts = 1;
  if (S == 0) return TP_OK;
  const int Hl = nh * d;    // columns of the heads held here
  const int Hs = Hl / t;    // columns of one shard's heads
  GemmExtra ex;  // scratch for stream-K partials (its plan never also splits K into slots)
  ex.sk_ws = sk_ws;
  ex.sk_ws_bytes = sk_bytes;
  // [Q_s | K_s | V_s] = in Wqkv_s into columns [3 s Hs, 3 (s+1) Hs) of QKV.
  int st = run_gemm_tc(dev, in, H, S, Wqkv_shards, t, 0, H, 3 * Hs, QKV, 3LL * Hl, 0, TP_ACT_NONE, s, 1, 0, nullptr,
                       kmaj, &ex);
  if (st != TP_OK) return st;
  // O_h = softmax(Q_h K_h^T / sqrt d) V_h, written to columns [h d, (h+1) d) of O.
  {
    tp::AttnArgs a;
    std::memset(&a, 0, sizeof(a));
    const int nhs = nh / t;
    // Q/K/V boxes: 64 columns (128 B) x 128 rows of the [S, 3 Hl] buffer.
    if (!tmap_bf16(&a.tmQKV, QKV, S, 3LL * Hl, 3LL * Hl, 64, tp::attn::BQ)) return TP_ERR_CUDA;
    a.O = Obuf;
    a.S = S;
    a.H = Hl;
    a.nh = nh;
    a.heads_per_shard = nhs;
    a.shard_cols = 3 * Hs;
    a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
    a.lse2 = lse2;
    a.nq = (S + tp::attn::TILES * tp::attn::BQ - 1) / (tp::attn::TILES * tp::attn::BQ);
    // The key-split scratch is the partial-sum area, which the O projection
    // below overwrites only after this kernel.
    const AttnSplit sp = attn_split_plan(S, nh, dev.sm_count, g_attn_split, zsum_bytes);
    a.whole = sp.whole;
    a.kv_half = sp.kv_half;
    if (sp.split > 0) {
      uint8_t* w = reinterpret_cast<uint8_t*>(Zsum);
      const size_t ob = align256(static_cast<size_t>(sp.split) * 8 * 32 * tp::attn::D * 4);
      a.part_o = reinterpret_cast<float*>(w);
      a.part_ml = reinterpret_cast<float*>(w + ob);
      a.part_flags = reinterpret_cast<unsigned long long*>(w + ob + align256(static_cast<size_t>(sp.split) * 8 * 64 * 4));
      a.epoch = next_sk_epoch();
    }
    dim3 grid(sp.whole + 2 * sp.split);
    ProfScope ps(K_ATTN, s);
    st = launch_pdl(tp::attn_fwd_kernel, grid, dim3(tp::attn::NUM_THREADS), tp::attn::SMEM_BYTES, s, a) != cudaSuccess
             ? TP_ERR_CUDA
             : launch_status();
    if (st != TP_OK) return st;
  }
  // sum_s O_s Wo_s, the O projection row-split by head, summed in TMEM.
  return run_gemm_tc(dev, Obuf, Hl, S, Wo_shards, t, 1, Hs, H, Zsum, H, 1, TP_ACT_NONE, s, max_splits,
                     static_cast<long long>(S) * H, nparts, kmaj, &ex);
}

int attn_core(const DeviceInfo& dev, int S, int H, int nh, int d, int t, int out_dtype, const void* in,
              const void* res, const void* const* Wqkv_shards, const void* const* Wo_shards, const float* gamma,
              const float* beta, float eps, int apply_ln, void* Y, void* workspace, cudaStream_t s,
              int kmaj = 0, const AttnKeep* keep = nullptr) {
  if (S == 0) return TP_OK;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* QKV = keep ? keep->qkv : ws;                                         // [S, 3H] bf16
  void* Obuf = keep ? keep->o : ws + align256(static_cast<size_t>(S) * 3 * H * 2);   // [S, H] bf16
  float* Zsum = keep ? keep->zsum
                     : reinterpret_cast<float*>(static_cast<uint8_t*>(Obuf) + align256(static_cast<size_t>(S) * H * 2));
  int nparts = 1;
  // Slots 1.. of the partial-sum area double as stream-K scratch (not when a
  // training forward keeps a single slot in its state).
  const size_t sh4 = static_cast<size_t>(S) * H * 4;
  int st = attn_products(dev, S, H, nh, d, t, in, Wqkv_shards, Wo_shards, QKV, Obuf, Zsum,
                         keep ? 1 : TP_MAX_K_SPLITS, &nparts, s, kmaj, keep ? keep->lse2 : nullptr,
                         keep ? nullptr : reinterpret_cast<uint8_t*>(Zsum) + sh4, keep ? 0 : (TP_MAX_K_SPLITS - 1) * sh4,
                         keep ? sh4 : TP_MAX_K_SPLITS * sh4);
  if (st != TP_OK) return st;
  return run_reduce_ln(S, H, nparts, Zsum, res, 1, gamma, beta, eps, Y, out_dtype == TP_DTYPE_BF16, s, dev.sm_count,
                       apply_ln, nullptr, 0, nullptr, keep ? keep->stats : nullptr);
}

int check_mlp_args(int S, int H, int F, int t, int dtype, int out_dtype, const void* X, const void* const* A_shards,
                   const void* const* B_shards, const float* gamma, const float* beta, float eps, int act,
                   const void* Y) {
  if (t < 1 || t > TP_MAX_SHARDS || S < 0 || H <= 0 || F <= 0) return TP_ERR_INVALID_ARG;
  if (!valid_out(dtype, out_dtype) || !valid_act(act) || !(eps > 0.0f) || !std::isfinite(eps))
    return TP_ERR_INVALID_ARG;
  // With S == 0 nothing is read or written, so X and Y may be null.
  if ((S > 0 && (!ptr_ok(X) || !ptr_ok(Y))) || !opt_ptr_ok(X) || !opt_ptr_ok(Y) || !shards_ok(A_shards, t) ||
      !shards_ok(B_shards, t) || !opt_ptr_ok(gamma) || !opt_ptr_ok(beta))
    return TP_ERR_INVALID_ARG;
  if (F % t != 0 || (F / t) % 8 != 0 || !hidden_ok(H)) return TP_ERR_UNSUPPORTED_SHAPE;
  return TP_OK;
}

int check_attn_args(int S, int H, int nh, int d, int t, int dtype, int out_dtype, const void* X,
                    const void* const* Wqkv_shards, const void* const* Wo_shards, const float* gamma,
                    const float* beta, float eps, const void* Y) {
  if (t < 1 || t > TP_MAX_SHARDS || S < 0 || H <= 0 || nh <= 0 || d <= 0) return TP_ERR_INVALID_ARG;
  if (dtype != TP_DTYPE_BF16 || !valid_out(dtype, out_dtype) || !(eps > 0.0f) || !std::isfinite(eps))
    return TP_ERR_INVALID_ARG;
  if ((S > 0 && (!ptr_ok(X) || !ptr_ok(Y))) || !opt_ptr_ok(X) || !opt_ptr_ok(Y) || !shards_ok(Wqkv_shards, t) ||
      !shards_ok(Wo_shards, t) || !opt_ptr_ok(gamma) || !opt_ptr_ok(beta))
    return TP_ERR_INVALID_ARG;
  if (d != tp::attn::D || static_cast<long long>(nh) * d != H || nh % t != 0 || S % tp::attn::BQ != 0 ||
      !hidden_ok(H))
    return TP_ERR_UNSUPPORTED_SHAPE;
  return TP_OK;
}

}  // namespace

int tp_internal_check_mlp_args(int S, int H, int F, int t, int dtype, int out_dtype, const void* X,
                               const void* const* A_shards, const void* const* B_shards, const float* gamma,
                               const float* beta, float eps, int act, const void* Y) {
  return check_mlp_args(S, H, F, t, dtype, out_dtype, X, A_shards, B_shards, gamma, beta, eps, act, Y);
}

extern "C" {

int tp_mlp_forward(int S, int H, int F, int t, int dtype, int out_dtype, const void* X,
                   const void* const* A_shards, const void* const* B_shards, const float* gamma,
                   const float* beta, float eps, int act, void* Y, void* workspace, size_t workspace_bytes,
                   void* stream) {
  return tp_mlp_forward_ex(S, H, F, t, dtype, out_dtype, TP_W_IN_OUT, X, A_shards, B_shards, gamma, beta, eps, act, Y,
                           workspace, workspace_bytes, stream);
}

int tp_mlp_forward_ex(int S, int H, int F, int t, int dtype, int out_dtype, int w_layout, const void* X,
                      const void* const* A_shards, const void* const* B_shards, const float* gamma,
                      const float* beta, float eps, int act, void* Y, void* workspace, size_t workspace_bytes,
                      void* stream) {
  if (w_layout != TP_W_IN_OUT && w_layout != TP_W_OUT_IN) return TP_ERR_INVALID_ARG;
  int st = check_mlp_args(S, H, F, t, dtype, out_dtype, X, A_shards, B_shards, gamma, beta, eps, act, Y);
  if (st != TP_OK) return st;
  if (!opt_ptr_ok(workspace)) return TP_ERR_INVALID_ARG;
  const size_t need = tp_mlp_workspace_bytes(S, H, F, t, dtype);
  if (workspace_bytes < need || (need > 0 && !workspace)) return TP_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  st = device_ready(&dev);
  if (st != TP_OK) return st;
  return mlp_core(*dev, S, H, F, t, dtype, out_dtype, X, X, A_shards, B_shards, gamma, beta, eps, act, 1, Y,
                  workspace, static_cast<cudaStream_t>(stream), w_layout == TP_W_OUT_IN);
}

// ------------------------------------------------------- MLP training step
size_t tp_mlp_train_state_bytes(int S, int H, int F, int t, int dtype) {
  if (S < 0 || H <= 0 || F <= 0 || t < 1 || dtype != TP_DTYPE_BF16) return 0;
  return train_state_layout(S, H, F).bytes;
}

int tp_mlp_forward_train(int S, int H, int F, int t, int dtype, int out_dtype, const void* X,
                         const void* const* A_shards, const void* const* B_shards, const float* gamma,
                         const float* beta, float eps, int act, void* Y, void* state, size_t state_bytes,
                         void* stream) {
  return tp_mlp_forward_train_ex(S, H, F, t, dtype, out_dtype, TP_W_IN_OUT, X, A_shards, B_shards, gamma, beta, eps,
                                 act, Y, state, state_bytes, stream);
}

int tp_mlp_forward_train_ex(int S, int H, int F, int t, int dtype, int out_dtype, int w_layout, const void* X,
                            const void* const* A_shards, const void* const* B_shards, const float* gamma,
                            const float* beta, float eps, int act, void* Y, void* state, size_t state_bytes,
                            void* stream) {
  if (w_layout != TP_W_IN_OUT && w_layout != TP_W_OUT_IN) return TP_ERR_INVALID_ARG;
  if (dtype != TP_DTYPE_BF16) return TP_ERR_UNSUPPORTED_SHAPE;
  int st = check_mlp_args(S, H, F, t, dtype, out_dtype, X, A_shards, B_shards, gamma, beta, eps, act, Y);
  if (st != TP_OK) return st;
  if (!opt_ptr_ok(state)) return TP_ERR_INVALID_ARG;
  if (S == 0) return TP_OK;
  const TrainState L = train_state_layout(S, H, F);
  if (!state || state_bytes < L.bytes) return TP_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  st = device_ready(&dev);
  if (st != TP_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(state);
  void* U = base + L.off_u;
  void* G = base + L.off_g;
  float* V = reinterpret_cast<float*>(base + L.off_v);
  const int Fs = F / t;
  // G_i = Act(X A_i) into columns [i Fs, (i+1) Fs) of G, and U_i = X A_i (the
  // pre-activation, from the same accumulator) into the same columns of U.
  GemmExtra ex;
  ex.epi_mode = tp::EPI_AUX_PRE;
  ex.aux = U;
  ex.ld_aux = F;
  const int kmaj = w_layout == TP_W_OUT_IN;
  st = run_gemm_tc(*dev, X, H, S, A_shards, t, 0, H, Fs, G, F, 0, act, s, 1, 0, nullptr, kmaj, &ex);
  if (st != TP_OK) return st;
  // V = sum_i G_i B_i in one f32 slot (no K split: the backward reads one).
  st = run_gemm_tc(*dev, G, F, S, B_shards, t, 1, Fs, H, V, H, 1, TP_ACT_NONE, s, 1, 0, nullptr, kmaj);
  if (st != TP_OK) return st;
  return run_reduce_ln(S, H, 1, V, X, 1, gamma, beta, eps, Y, out_dtype == TP_DTYPE_BF16, s, dev->sm_count, 1,
                       nullptr, 0, nullptr, reinterpret_cast<float*>(base + L.off_stats));
}

size_t tp_mlp_backward_workspace_bytes(int S, int H, int F, int t, int dtype) {
  if (S < 0 || H <= 0 || F <= 0 || t < 1 || dtype != TP_DTYPE_BF16) return 0;
  return back_ws_layout(S, H, F).bytes;
}

int tp_mlp_backward(int S, int H, int F, int t, int dtype, const void* X, const void* const* A_shards,
                    const void* const* B_shards, const float* gamma, float eps, int act, const void* state,
                    size_t state_bytes, const void* dY, void* dX, void* const* dA_shards, void* const* dB_shards,
                    float* dgamma, float* dbeta, void* workspace, size_t workspace_bytes, void* stream) {
  return tp_mlp_backward_ex(S, H, F, t, dtype, TP_W_IN_OUT, X, A_shards, B_shards, gamma, eps, act, state,
                            state_bytes, dY, dX, dA_shards, dB_shards, dgamma, dbeta, workspace, workspace_bytes,
                            stream);
}

int tp_mlp_backward_ex(int S, int H, int F, int t, int dtype, int w_layout, const void* X,
                       const void* const* A_shards, const void* const* B_shards, const float* gamma, float eps,
                       int act, const void* state, size_t state_bytes, const void* dY, void* dX,
                       void* const* dA_shards, void* const* dB_shards, float* dgamma, float* dbeta, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (w_layout != TP_W_IN_OUT && w_layout != TP_W_OUT_IN) return TP_ERR_INVALID_ARG;
  if (dtype != TP_DTYPE_BF16) return TP_ERR_UNSUPPORTED_SHAPE;
  int st = check_mlp_args(S, H, F, t, dtype, TP_DTYPE_BF16, X, A_shards, B_shards, gamma, nullptr, eps, act, dX);
  if (st != TP_OK) return st;
  if ((S > 0 && (!ptr_ok(dY) || !ptr_ok(state))) || !opt_ptr_ok(dY) || !opt_ptr_ok(state) ||
      !shards_ok(dA_shards, t) || !shards_ok(dB_shards, t) || !opt_ptr_ok(dgamma) || !opt_ptr_ok(dbeta) ||
      !opt_ptr_ok(workspace))
    return TP_ERR_INVALID_ARG;
  if (S == 0) return TP_OK;  // weight gradients of an empty batch: the caller's buffers are left as they are
  if (state_bytes < train_state_layout(S, H, F).bytes) return TP_ERR_WORKSPACE_TOO_SMALL;
  const BackWs W = back_ws_layout(S, H, F);
  if (!workspace || workspace_bytes < W.bytes) return TP_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  st = device_ready(&dev);
  if (st != TP_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const TrainState L = train_state_layout(S, H, F);
  const uint8_t* sb = static_cast<const uint8_t*>(state);
  const void* U = sb + L.off_u;
  const uint8_t* G = sb + L.off_g;
  const float* V = reinterpret_cast<const float*>(sb + L.off_v);
  uint8_t* wb = static_cast<uint8_t*>(workspace);
  void* dZ = wb + W.off_dz;
  uint8_t* dU = wb + W.off_du;
  float* dXp = reinterpret_cast<float*>(wb + W.off_dxp);
  float* part = reinterpret_cast<float*>(wb + W.off_part);
  const int Fs = F / t;
  // 1. Through the LayerNorm: dZ, dgamma, dbeta.
  const float* stats = reinterpret_cast<const float*>(sb + L.off_stats);
  st = run_ln_backward(S, H, V, stats, X, dY, gamma, dZ, part, dgamma, dbeta, s, dev->sm_count);
  if (st != TP_OK) return st;
  // In [out, in] storage (TP_W_OUT_IN) every weight is the transpose of its
  // [in, out] form: the backward reads B_i and A_i with the other majorness,
  // and each weight gradient is the transpose of the [in, out] one, computed
  // with the operands' roles swapped (dA_i^T = dU_i^T X, dB_i^T = dZ^T G_i).
  const bool oi = w_layout == TP_W_OUT_IN;
  // 2. Through V = G B and G = Act(U): dU_i = (dZ B_i^T) * Act'(U_i) into the
  //    columns of shard i.
  {
    GemmExtra ex;
    ex.epi_mode = tp::EPI_GRAD;
    ex.aux = U;
    ex.ld_aux = F;
    st = run_gemm_tc(*dev, dZ, H, S, B_shards, t, 0, H, Fs, dU, F, 0, act, s, 1, 0, nullptr, oi ? 0 : 1, &ex);
    if (st != TP_OK) return st;
  }
  // 3. Through U = X A and the residual: dX = dZ + sum_i dU_i A_i^T (row split
  //    over the shards), then the residual add.
  st = run_gemm_tc(*dev, dU, F, S, A_shards, t, 1, Fs, H, dXp, H, 1, TP_ACT_NONE, s, 1, 0, nullptr, oi ? 0 : 1);
  if (st != TP_OK) return st;
  st = run_reduce_ln(S, H, 1, dXp, dZ, 1, nullptr, nullptr, 1.0f, dX, 1, s, dev->sm_count, /*apply_ln=*/0);
  if (st != TP_OK) return st;
  // 4. Weight gradients, each with its own shard.  A column-mode launch on an
  //    M-major A operand with strided B shards, or an M-split launch (all
  //    shards' rows in one GEMM) when F/t is a multiple of 256, else one
  //    launch per shard.
  //    [in, out]: dA_i = X^T dU_i (column mode over dU's slices),
  //               dB_i = G_i^T dZ (M-split over G's columns).
  //    [out, in]: dB_i^T = dZ^T G_i (column mode over G's slices),
  //               dA_i^T = dU_i^T X (M-split over dU's columns).
  const uint8_t* colsrc = oi ? G : dU;     // the column-mode launch's strided B shards
  const void* colA = oi ? dZ : X;          // ... and its M-major A ([S, H])
  void* const* colOut = oi ? dB_shards : dA_shards;
  const uint8_t* splitA = oi ? dU : G;     // the M-split launch's M-major A ([S, F])
  const void* splitB = oi ? X : dZ;        // ... and its B ([S, H])
  void* const* splitOut = oi ? dA_shards : dB_shards;
  {
    const void* sh[TP_MAX_SHARDS];
    for (int i = 0; i < t; ++i) sh[i] = colsrc + static_cast<size_t>(i) * Fs * 2;
    GemmExtra ex;
    ex.a_mnmajor = 1;
    ex.ldb = F;
    ex.C_shards = colOut;
    ex.ldc_shard = Fs;
    st = run_gemm_tc(*dev, colA, H, H, sh, t, 0, S, Fs, nullptr, Fs, 1, TP_ACT_NONE, s, 1, 0, nullptr, 0, &ex);
    if (st != TP_OK) return st;
  }
  const void* b1[1] = {splitB};
  if (t > 1 && Fs % 256 == 0) {  // F >= 512 rows: the CTA-pair GEMM with 256-row tiles
    GemmExtra ex;
    ex.a_mnmajor = 1;
    ex.n_fastest = TP_DB_N_FASTEST;  // G (S x F) is read once per wave, not once per column block
    ex.m_split = t;
    ex.C_shards = splitOut;
    ex.ldc_shard = H;
    return run_gemm_tc(*dev, splitA, F, F, b1, 1, 0, S, H, nullptr, H, 1, TP_ACT_NONE, s, 1, 0, nullptr, 0, &ex);
  }
  for (int i = 0; i < t; ++i) {
    GemmExtra ex;
    ex.a_mnmajor = 1;
    ex.n_fastest = TP_DB_N_FASTEST;
    st = run_gemm_tc(*dev, splitA + static_cast<size_t>(i) * Fs * 2, F, Fs, b1, 1, 0, S, H, splitOut[i], H, 1,
                     TP_ACT_NONE, s, 1, 0, nullptr, 0, &ex);
    if (st != TP_OK) return st;
  }
  return TP_OK;
}

// -------------------------------------------------------------- attention
size_t tp_attn_workspace_bytes(int S, int H, int nh, int d, int t, int dtype) {
  if (S < 0 || H <= 0 || nh <= 0 || d <= 0 || t < 1 || dtype != TP_DTYPE_BF16) return 0;
  const size_t s = static_cast<size_t>(S), h = static_cast<size_t>(H);
  return align256(s * 3 * h * 2) + align256(s * h * 2) + TP_MAX_K_SPLITS * s * h * 4;
}

int tp_qkv_attn_oproj_forward(int S, int H, int nh, int d, int t, int dtype, int out_dtype, const void* X,
                              const void* const* Wqkv_shards, const void* const* Wo_shards, const float* gamma,
                              const float* beta, float eps, void* Y, void* workspace, size_t workspace_bytes,
                              void* stream) {
  return tp_qkv_attn_oproj_forward_ex(S, H, nh, d, t, dtype, out_dtype, TP_W_IN_OUT, X, Wqkv_shards, Wo_shards, gamma,
                                      beta, eps, Y, workspace, workspace_bytes, stream);
}

int tp_qkv_attn_oproj_forward_ex(int S, int H, int nh, int d, int t, int dtype, int out_dtype, int w_layout,
                                 const void* X, const void* const* Wqkv_shards, const void* const* Wo_shards,
                                 const float* gamma, const float* beta, float eps, void* Y, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (w_layout != TP_W_IN_OUT && w_layout != TP_W_OUT_IN) return TP_ERR_INVALID_ARG;
  int st = check_attn_args(S, H, nh, d, t, dtype, out_dtype, X, Wqkv_shards, Wo_shards, gamma, beta, eps, Y);
  if (st != TP_OK) return st;
  if (!opt_ptr_ok(workspace)) return TP_ERR_INVALID_ARG;
  const size_t need = tp_attn_workspace_bytes(S, H, nh, d, t, dtype);
  if (workspace_bytes < need || (need > 0 && !workspace)) return TP_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  st = device_ready(&dev);
  if (st != TP_OK) return st;
  return attn_core(*dev, S, H, nh, d, t, out_dtype, X, X, Wqkv_shards, Wo_shards, gamma, beta, eps, 1, Y, workspace,
                   static_cast<cudaStream_t>(stream), w_layout == TP_W_OUT_IN);
}

// ---------------------------------------------------------- Transformer block
// ------------------------------------------------- attention training step
namespace {
struct AttnState {
  size_t off_qkv, off_o, off_z, off_lse, off_stats, bytes;
};
AttnState attn_state_layout(int S, int H, int nh) {
  AttnState a;
  const size_t s = static_cast<size_t>(S), h = static_cast<size_t>(H);
  a.off_qkv = 0;
  a.off_o = align256(s * 3 * h * 2);
  a.off_z = a.off_o + align256(s * h * 2);
  a.off_lse = a.off_z + align256(s * h * 4);
  a.off_stats = a.off_lse + align256(static_cast<size_t>(nh) * s * 4);
  a.bytes = a.off_stats + align256(s * 8);
  return a;
}
struct AttnBackWs {
  size_t off_dz, off_do, off_dqkv, off_dxp, off_p, off_ds, off_d, off_part, bytes;
};
// Heads whose [S, S] P and dS matrices (bf16, 4 bytes an element for the
// two) the backward holds at once: as many as one GEMM launch takes
// (MAX_SHARDS), fewer where that would pass 1 GiB.
int attn_back_group(int S, int nh) {
  int g = nh < MAX_SHARDS ? nh : MAX_SHARDS;
  const size_t per_head = static_cast<size_t>(S) * S * 4;
  while (g > 1 && per_head * g > (static_cast<size_t>(1) << 30)) --g;
  return g;
}
AttnBackWs attn_back_layout(int S, int H, int nh) {
  AttnBackWs w;
  const size_t s = static_cast<size_t>(S), h = static_cast<size_t>(H);
  // P and dS in memory only for the per-head GEMM form.
  const size_t ss = TP_ATTN_BACK_FUSED ? 0 : static_cast<size_t>(attn_back_group(S, nh)) * s * s;
  w.off_dz = 0;
  w.off_do = align256(s * h * 2);
  w.off_dqkv = w.off_do + align256(s * h * 2);
  w.off_dxp = w.off_dqkv + align256(s * 3 * h * 2);
  w.off_p = w.off_dxp + align256(s * h * 4);
  w.off_ds = w.off_p + align256(ss * 2);
  w.off_d = w.off_ds + align256(ss * 2);
  w.off_part = w.off_d + align256(static_cast<size_t>(nh) * s * 4);
  w.bytes = w.off_part + align256(static_cast<size_t>(LNB_MAX_CTAS) * 2 * h * 4);
  return w;
}
}  // namespace

size_t tp_attn_train_state_bytes(int S, int H, int nh, int d, int t, int dtype) {
  if (S < 0 || H <= 0 || nh <= 0 || d <= 0 || t < 1 || dtype != TP_DTYPE_BF16) return 0;
  return attn_state_layout(S, H, nh).bytes;
}

int tp_attn_forward_train(int S, int H, int nh, int d, int t, int dtype, int out_dtype, const void* X,
                          const void* const* Wqkv_shards, const void* const* Wo_shards, const float* gamma,
                          const float* beta, float eps, void* Y, void* state, size_t state_bytes, void* stream) {
  int st = check_attn_args(S, H, nh, d, t, dtype, out_dtype, X, Wqkv_shards, Wo_shards, gamma, beta, eps, Y);
  if (st != TP_OK) return st;
  if (!opt_ptr_ok(state)) return TP_ERR_INVALID_ARG;
  if (S == 0) return TP_OK;
  const AttnState L = attn_state_layout(S, H, nh);
  if (!state || state_bytes < L.bytes) return TP_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  st = device_ready(&dev);
  if (st != TP_OK) return st;
  uint8_t* b = static_cast<uint8_t*>(state);
  AttnKeep keep;
  keep.qkv = b + L.off_qkv;
  keep.o = b + L.off_o;
  keep.zsum = reinterpret_cast<float*>(b + L.off_z);
  keep.lse2 = reinterpret_cast<float*>(b + L.off_lse);
  keep.stats = reinterpret_cast<float*>(b + L.off_stats);
  return attn_core(*dev, S, H, nh, d, t, out_dtype, X, X, Wqkv_shards, Wo_shards, gamma, beta, eps, 1, Y, nullptr,
                   static_cast<cudaStream_t>(stream), 0, &keep);
}

size_t tp_attn_backward_workspace_bytes(int S, int H, int nh, int d, int t, int dtype) {
  if (S < 0 || H <= 0 || nh <= 0 || d <= 0 || t < 1 || dtype != TP_DTYPE_BF16) return 0;
  return attn_back_layout(S, H, nh).bytes;
}

int tp_attn_backward(int S, int H, int nh, int d, int t, int dtype, const void* X,
                     const void* const* Wqkv_shards, const void* const* Wo_shards, const float* gamma, float eps,
                     const void* state, size_t state_bytes, const void* dY, void* dX, void* const* dWqkv_shards,
                     void* const* dWo_shards, float* dgamma, float* dbeta, void* workspace, size_t workspace_bytes,
                     void* stream) {
  int st = check_attn_args(S, H, nh, d, t, dtype, TP_DTYPE_BF16, X, Wqkv_shards, Wo_shards, gamma, nullptr, eps, dX);
  if (st != TP_OK) return st;
  if ((S > 0 && (!ptr_ok(dY) || !ptr_ok(state))) || !opt_ptr_ok(dY) || !opt_ptr_ok(state) ||
      !shards_ok(dWqkv_shards, t) || !shards_ok(dWo_shards, t) || !opt_ptr_ok(dgamma) || !opt_ptr_ok(dbeta) ||
      !opt_ptr_ok(workspace))
    return TP_ERR_INVALID_ARG;
  if (S == 0) return TP_OK;
  const AttnState L = attn_state_layout(S, H, nh);
  if (state_bytes < L.bytes) return TP_ERR_WORKSPACE_TOO_SMALL;
  const AttnBackWs W = attn_back_layout(S, H, nh);
  if (!workspace || workspace_bytes < W.bytes) return TP_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  st = device_ready(&dev);
  if (st != TP_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int Hs = H / t, hps = nh / t;
  const long long H3 = 3LL * H;
  const uint8_t* sb = static_cast<const uint8_t*>(state);
  const uint8_t* QKV = sb + L.off_qkv;
  const uint8_t* Ob = sb + L.off_o;
  const float* Vo = reinterpret_cast<const float*>(sb + L.off_z);
  const float* lse2 = reinterpret_cast<const float*>(sb + L.off_lse);
  uint8_t* wb = static_cast<uint8_t*>(workspace);
  void* dZ = wb + W.off_dz;
  uint8_t* dO = wb + W.off_do;
  uint8_t* dQKV = wb + W.off_dqkv;
  float* dXp = reinterpret_cast<float*>(wb + W.off_dxp);
#if !TP_ATTN_BACK_FUSED
  __nv_bfloat16* P = reinterpret_cast<__nv_bfloat16*>(wb + W.off_p);
  __nv_bfloat16* dS = reinterpret_cast<__nv_bfloat16*>(wb + W.off_ds);
#endif
  float* D = reinterpret_cast<float*>(wb + W.off_d);
  float* part = reinterpret_cast<float*>(wb + W.off_part);
  // 1. Through the LayerNorm: dZ, dgamma, dbeta (Z = X + the O projection's output).
  const float* stats = reinterpret_cast<const float*>(sb + L.off_stats);
  st = run_ln_backward(S, H, Vo, stats, X, dY, gamma, dZ, part, dgamma, dbeta, s, dev->sm_count);
  if (st != TP_OK) return st;
  // 2. Through the O projection: dO_s = dZ Wo_s^T (Wo_s [Hs, H] read K-major)
  //    into shard s's head columns of dO, and dWo_s = O_s^T dZ.
  st = run_gemm_tc(*dev, dZ, H, S, Wo_shards, t, 0, H, Hs, dO, H, 0, TP_ACT_NONE, s, 1, 0, nullptr, 1);
  if (st != TP_OK) return st;
  {
    const void* b1[1] = {dZ};
    if (t > 1 && Hs % 256 == 0) {
      GemmExtra ex;
      ex.a_mnmajor = 1;
      ex.m_split = t;
      ex.C_shards = dWo_shards;
      ex.ldc_shard = H;
      st = run_gemm_tc(*dev, Ob, H, H, b1, 1, 0, S, H, nullptr, H, 1, TP_ACT_NONE, s, 1, 0, nullptr, 0, &ex);
      if (st != TP_OK) return st;
    } else {
      for (int i = 0; i < t; ++i) {
        GemmExtra ex;
        ex.a_mnmajor = 1;
        st = run_gemm_tc(*dev, Ob + static_cast<size_t>(i) * Hs * 2, H, Hs, b1, 1, 0, S, H, dWo_shards[i], H, 1,
                         TP_ACT_NONE, s, 1, 0, nullptr, 0, &ex);
        if (st != TP_OK) return st;
      }
    }
  }
  // 3. Through the softmax attention of every head: D_h = rowsum(dO_h * O_h)
  //    for all heads, then the heads in groups (P rebuilt from the scores and
  //    the forward's log2 denominators).
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  const float scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  {
  ProfScope ps(K_ATTN_BACK, s);
  st = launch_pdl(tp::rowdot_kernel, dim3(ceil_div(static_cast<long long>(S) * nh * 32, 256 * tp::ROWDOT_ITEMS)),
                  dim3(256), 0, s,
                  reinterpret_cast<const __nv_bfloat16*>(dO), reinterpret_cast<const __nv_bfloat16*>(Ob), D, S, H,
                  nh) != cudaSuccess
           ? TP_ERR_CUDA
           : launch_status();
  }
  if (st != TP_OK) return st;
#if TP_ATTN_BACK_FUSED
  // Every head at once: dV and dK from the key-major kernel, dQ from the
  // query-major one, straight into their columns of dQKV.
  {
    tp::AttnBwdArgs ab;
    std::memset(&ab, 0, sizeof(ab));
    if (!tmap_bf16(&ab.tmQKV_t, QKV, S, H3, H3, 64, tp::attb::BT) ||
        !tmap_bf16(&ab.tmQKV_s, QKV, S, H3, H3, 64, tp::attb::BS) ||
        !tmap_bf16(&ab.tmdO_t, dO, S, H, H, 64, tp::attb::BT) ||
        !tmap_bf16(&ab.tmdO_s, dO, S, H, H, 64, tp::attb::BS))
      return TP_ERR_CUDA;
    ab.lse2 = lse2;
    ab.Dvec = D;
    ab.dQKV = reinterpret_cast<__nv_bfloat16*>(dQKV);
    ab.ld_qkv = H3;
    ab.S = S;
    ab.nh = nh;
    ab.heads_per_shard = hps;
    ab.shard_cols = 3 * Hs;
    ab.scale_log2 = scale_log2;
    ab.scale = scale;
    const dim3 grid(S / tp::attb::BT, nh);
    {
      ProfScope ps(K_ATTN_BWD, s);
      if (launch_pdl(tp::attn_bwd_dkv_kernel, grid, dim3(tp::attb::DKV_THREADS), tp::attb::SMEM_DKV, s, ab) !=
          cudaSuccess)
        return TP_ERR_CUDA;
    }
    {
      ProfScope ps(K_ATTN_BWD, s);
      if (launch_pdl(tp::attn_bwd_dq_kernel, grid, dim3(tp::attb::DQ_THREADS), tp::attb::SMEM_DQ, s, ab) !=
          cudaSuccess)
        return TP_ERR_CUDA;
    }
    st = launch_status();
    if (st != TP_OK) return st;
  }
#else
  // The heads go through in groups of G: each GEMM below is one launch over
  // the group's heads (shard j of the launch = head h0 + j, with its own A, B
  // and output).  P and dS are [S, G S] with head j in columns [j S, (j+1) S);
  // the softmax and its backward run in the epilogues of the GEMMs that make
  // the scores and dP, so neither f32 matrix reaches memory.
  const int G = attn_back_group(S, nh);
  const long long GS = static_cast<long long>(G) * S;
  for (int h0 = 0; h0 < nh; h0 += G) {
    const int g = nh - h0 < G ? nh - h0 : G;
    const void *Qg[MAX_SHARDS], *Kg[MAX_SHARDS], *Vg[MAX_SHARDS], *dOg[MAX_SHARDS], *Pg[MAX_SHARDS],
        *dSg[MAX_SHARDS];
    void *dQg[MAX_SHARDS], *dKg[MAX_SHARDS], *dVg[MAX_SHARDS];
    for (int j = 0; j < g; ++j) {
      const int h = h0 + j, sh = h / hps, hj = h % hps;
      const long long qcol = static_cast<long long>(sh) * 3 * Hs + static_cast<long long>(hj) * d;
      Qg[j] = QKV + qcol * 2;
      Kg[j] = QKV + (qcol + Hs) * 2;
      Vg[j] = QKV + (qcol + 2LL * Hs) * 2;
      dOg[j] = dO + static_cast<long long>(h) * d * 2;
      Pg[j] = P + static_cast<long long>(j) * S;
      dSg[j] = dS + static_cast<long long>(j) * S;
      dQg[j] = dQKV + qcol * 2;
      dKg[j] = dQKV + (qcol + Hs) * 2;
      dVg[j] = dQKV + (qcol + 2LL * Hs) * 2;
    }
#if TP_ATTN_BACK_DUAL
    // P_h = 2^(Q_h K_h^T scale_log2 - lse2_h) and dS_h = P_h (dO_h V_h^T - D_h) / sqrt d
    // from one tile: the scores and dP of the same 256 x 256 block in the two
    // halves of TMEM (K_h and V_h [keys, d] are the K-major B operands).
    {
      GemmExtra ex;
      ex.ldb = H3;
      ex.A_shards = Qg;
      ex.A2_shards = dOg;
      ex.lda2 = H;
      ex.B2_shards = Vg;
      ex.ldb2 = H3;
      ex.epi_mode = tp::EPI_DUAL_SOFTMAX;
      ex.aux = dS;
      ex.ld_aux = GS;
      ex.rowvec = lse2 + static_cast<long long>(h0) * S;
      ex.rowvec2 = D + static_cast<long long>(h0) * S;
      ex.rowvec_ld = S;
      ex.epi_scale = scale_log2;
      ex.epi_scale2 = scale;
      st = run_gemm_tc(*dev, Qg[0], H3, S, Kg, g, 0, d, S, P, GS, 0, TP_ACT_NONE, s, 1, 0, nullptr, 1, &ex);
      if (st != TP_OK) return st;
    }
#else
    // P_h = 2^(Q_h K_h^T scale_log2 - lse2_h) (K_h [keys, d] is the K-major B operand)
    {
      GemmExtra ex;
      ex.ldb = H3;
      ex.A_shards = Qg;
      ex.epi_mode = tp::EPI_SOFTMAX;
      ex.rowvec = lse2 + static_cast<long long>(h0) * S;
      ex.rowvec_ld = S;
      ex.epi_scale = scale_log2;
      st = run_gemm_tc(*dev, Qg[0], H3, S, Kg, g, 0, d, S, P, GS, 0, TP_ACT_NONE, s, 1, 0, nullptr, 1, &ex);
      if (st != TP_OK) return st;
    }
#endif
    // dV_h = P_h^T dO_h into V_h's columns of dQKV (P_h read M-major)
    {
      GemmExtra ex;
      ex.a_mnmajor = 1;
      ex.ldb = H;
      ex.A_shards = Pg;
      ex.C_shards = dVg;
      ex.ldc_shard = H3;
      st = run_gemm_tc(*dev, Pg[0], GS, S, dOg, g, 0, S, d, dVg[0], H3, 0, TP_ACT_NONE, s, 1, 0, nullptr, 0, &ex);
      if (st != TP_OK) return st;
    }
#if !TP_ATTN_BACK_DUAL
    // dS_h = P_h (dO_h V_h^T - D_h) / sqrt d (V_h [keys, d] is the K-major B operand)
    {
      GemmExtra ex;
      ex.ldb = H3;
      ex.A_shards = dOg;
      ex.epi_mode = tp::EPI_DSOFTMAX;
      ex.aux = P;
      ex.ld_aux = GS;
      ex.rowvec = D + static_cast<long long>(h0) * S;
      ex.rowvec_ld = S;
      ex.epi_scale = scale;
      st = run_gemm_tc(*dev, dOg[0], H, S, Vg, g, 0, d, S, dS, GS, 0, TP_ACT_NONE, s, 1, 0, nullptr, 1, &ex);
      if (st != TP_OK) return st;
    }
#endif
    // dQ_h = dS_h K_h and dK_h = dS_h^T Q_h into their columns of dQKV
    {
      GemmExtra ex;
      ex.ldb = H3;
      ex.A_shards = dSg;
      ex.C_shards = dQg;
      ex.ldc_shard = H3;
      st = run_gemm_tc(*dev, dSg[0], GS, S, Kg, g, 0, S, d, dQg[0], H3, 0, TP_ACT_NONE, s, 1, 0, nullptr, 0, &ex);
      if (st != TP_OK) return st;
    }
    {
      GemmExtra ex;
      ex.a_mnmajor = 1;
      ex.ldb = H3;
      ex.A_shards = dSg;
      ex.C_shards = dKg;
      ex.ldc_shard = H3;
      st = run_gemm_tc(*dev, dSg[0], GS, S, Qg, g, 0, S, d, dKg[0], H3, 0, TP_ACT_NONE, s, 1, 0, nullptr, 0, &ex);
      if (st != TP_OK) return st;
    }
  }
#endif
  // 4. Through the QKV projection and the residual: dX = dZ + sum_s dQKV_s
  //    Wqkv_s^T (row split over the shards, Wqkv_s [H, 3 Hs] read K-major),
  //    then dWqkv_s = X^T dQKV_s.
  st = run_gemm_tc(*dev, dQKV, H3, S, Wqkv_shards, t, 1, 3 * Hs, H, dXp, H, 1, TP_ACT_NONE, s, 1, 0, nullptr, 1);
  if (st != TP_OK) return st;
  st = run_reduce_ln(S, H, 1, dXp, dZ, 1, nullptr, nullptr, 1.0f, dX, 1, s, dev->sm_count, /*apply_ln=*/0);
  if (st != TP_OK) return st;
  {
    const void* sh[TP_MAX_SHARDS];
    for (int i = 0; i < t; ++i) sh[i] = dQKV + static_cast<size_t>(i) * 3 * Hs * 2;
    GemmExtra ex;
    ex.a_mnmajor = 1;
    ex.ldb = H3;
    ex.C_shards = dWqkv_shards;
    ex.ldc_shard = 3 * Hs;
    return run_gemm_tc(*dev, X, H, H, sh, t, 0, S, 3 * Hs, nullptr, 3 * Hs, 1, TP_ACT_NONE, s, 1, 0, nullptr, 0,
                       &ex);
  }
}

size_t tp_block_workspace_bytes(int S, int H, int F, int nh, int d, int t, int dtype) {
  if (S < 0 || H <= 0 || F <= 0 || nh <= 0 || d <= 0 || t < 1 || dtype != TP_DTYPE_BF16) return 0;
  const size_t a = tp_attn_workspace_bytes(S, H, nh, d, t, dtype);
  const size_t m = tp_mlp_workspace_bytes(S, H, F, t, dtype);
  const size_t core = align256(a > m ? a : m);
  const size_t act = align256(static_cast<size_t>(S) * H * 2);
  return core + 2 * act;
}

int tp_transformer_block_forward(int S, int H, int F, int nh, int d, int t, int dtype, int out_dtype, int pre_ln,
                                 const void* X, const void* const* Wqkv_shards, const void* const* Wo_shards,
                                 const void* const* A_shards, const void* const* B_shards, const float* ln1_gamma,
                                 const float* ln1_beta, const float* ln2_gamma, const float* ln2_beta, float eps,
                                 int act, void* Y, void* workspace, size_t workspace_bytes, void* stream) {
  return tp_transformer_block_forward_ex(S, H, F, nh, d, t, dtype, out_dtype, pre_ln, TP_W_IN_OUT, X, Wqkv_shards,
                                         Wo_shards, A_shards, B_shards, ln1_gamma, ln1_beta, ln2_gamma, ln2_beta, eps,
                                         act, Y, workspace, workspace_bytes, stream);
}

int tp_transformer_block_forward_ex(int S, int H, int F, int nh, int d, int t, int dtype, int out_dtype, int pre_ln,
                                    int w_layout, const void* X, const void* const* Wqkv_shards,
                                    const void* const* Wo_shards, const void* const* A_shards,
                                    const void* const* B_shards, const float* ln1_gamma, const float* ln1_beta,
                                    const float* ln2_gamma, const float* ln2_beta, float eps, int act, void* Y,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  if (pre_ln != 0 && pre_ln != 1) return TP_ERR_INVALID_ARG;
  if (w_layout != TP_W_IN_OUT && w_layout != TP_W_OUT_IN) return TP_ERR_INVALID_ARG;
  const int kmaj = w_layout == TP_W_OUT_IN;
  int st = check_attn_args(S, H, nh, d, t, dtype, TP_DTYPE_BF16, X, Wqkv_shards, Wo_shards, ln1_gamma, ln1_beta,
                           eps, Y);
  if (st != TP_OK) return st;
  st = check_mlp_args(S, H, F, t, dtype, out_dtype, X, A_shards, B_shards, ln2_gamma, ln2_beta, eps, act, Y);
  if (st != TP_OK) return st;
  if (!opt_ptr_ok(workspace)) return TP_ERR_INVALID_ARG;
  const size_t need = tp_block_workspace_bytes(S, H, F, nh, d, t, dtype);
  if (workspace_bytes < need || (need > 0 && !workspace)) return TP_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  st = device_ready(&dev);
  if (st != TP_OK) return st;
  if (S == 0) return TP_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t a = tp_attn_workspace_bytes(S, H, nh, d, t, dtype);
  const size_t m = tp_mlp_workspace_bytes(S, H, F, t, dtype);
  uint8_t* core = static_cast<uint8_t*>(workspace);
  uint8_t* buf1 = core + align256(a > m ? a : m);                    // [S, H] bf16
  uint8_t* buf2 = buf1 + align256(static_cast<size_t>(S) * H * 2);   // [S, H] bf16
  if (!pre_ln) {
    // Y1 = LN1(X + Attn(X));  Y = LN2(Y1 + MLP(Y1))
    st = attn_core(*dev, S, H, nh, d, t, TP_DTYPE_BF16, X, X, Wqkv_shards, Wo_shards, ln1_gamma, ln1_beta, eps, 1,
                   buf1, core, s, kmaj);
    if (st != TP_OK) return st;
    return mlp_core(*dev, S, H, F, t, dtype, out_dtype, buf1, buf1, A_shards, B_shards, ln2_gamma, ln2_beta, eps,
                    act, 1, Y, core, s, kmaj);
  }
  // h1 = LN1(X);  Z1 = X + Attn(h1);  h2 = LN2(Z1);  Y = Z1 + MLP(h2)
  st = run_reduce_ln(S, H, 0, nullptr, X, 1, ln1_gamma, ln1_beta, eps, buf1, 1, s, dev->sm_count, 1);
  if (st != TP_OK) return st;
  st = attn_core(*dev, S, H, nh, d, t, TP_DTYPE_BF16, buf1, X, Wqkv_shards, Wo_shards, nullptr, nullptr, eps, 0,
                 buf2, core, s, kmaj);
  if (st != TP_OK) return st;
  st = run_reduce_ln(S, H, 0, nullptr, buf2, 1, ln2_gamma, ln2_beta, eps, buf1, 1, s, dev->sm_count, 1);
  if (st != TP_OK) return st;
  return mlp_core(*dev, S, H, F, t, dtype, out_dtype, buf1, buf2, A_shards, B_shards, nullptr, nullptr, eps, act, 0,
                  Y, core, s, kmaj);
}

// ---------------------------------------------------------------- linears
int tp_linear_column_forward(int M, int K, int N, int t, int dtype, int out_dtype, const void* X,
                             const void* const* W_shards, int act, void* Y, void* stream) {
  return tp_linear_column_forward_ex(M, K, N, t, dtype, out_dtype, TP_W_IN_OUT, X, W_shards, act, Y, stream);
}

int tp_linear_column_forward_ex(int M, int K, int N, int t, int dtype, int out_dtype, int w_layout, const void* X,
                                const void* const* W_shards, int act, void* Y, void* stream) {
  if (t < 1 || t > TP_MAX_SHARDS || M < 0 || K <= 0 || N <= 0) return TP_ERR_INVALID_ARG;
  if (!valid_out(dtype, out_dtype) || !valid_act(act)) return TP_ERR_INVALID_ARG;
  if (w_layout != TP_W_IN_OUT && w_layout != TP_W_OUT_IN) return TP_ERR_INVALID_ARG;
  if ((M > 0 && (!ptr_ok(X) || !ptr_ok(Y))) || !opt_ptr_ok(X) || !opt_ptr_ok(Y) || !shards_ok(W_shards, t))
    return TP_ERR_INVALID_ARG;
  if (K % 8 != 0 || N % t != 0 || (N / t) % 8 != 0) return TP_ERR_UNSUPPORTED_SHAPE;
  DeviceInfo* dev = nullptr;
  int st = device_ready(&dev);
  if (st != TP_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int kmaj = w_layout == TP_W_OUT_IN;
  if (dtype == TP_DTYPE_BF16)
    return run_gemm_tc(*dev, X, K, M, W_shards, t, 0, K, N / t, Y, N, out_dtype == TP_DTYPE_F32, act, s, 1, 0, nullptr,
                       kmaj);
  return run_gemm_simt(static_cast<const float*>(X), K, M, W_shards, t, 0, K, N / t, static_cast<float*>(Y), N,
                       act, s, kmaj);
}

int tp_linear_row_forward(int M, int K, int N, int t, int dtype, int out_dtype, const void* X,
                          const void* const* W_shards, void* Y, void* workspace, size_t workspace_bytes,
                          void* stream) {
  return tp_linear_row_forward_ex(M, K, N, t, dtype, out_dtype, TP_W_IN_OUT, X, W_shards, Y, workspace,
                                  workspace_bytes, stream);
}

int tp_linear_row_forward_ex(int M, int K, int N, int t, int dtype, int out_dtype, int w_layout, const void* X,
                             const void* const* W_shards, void* Y, void* workspace, size_t workspace_bytes,
                             void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (t < 1 || t > TP_MAX_SHARDS || M < 0 || K <= 0 || N <= 0) return TP_ERR_INVALID_ARG;
  if (!valid_out(dtype, out_dtype)) return TP_ERR_INVALID_ARG;
  if (w_layout != TP_W_IN_OUT && w_layout != TP_W_OUT_IN) return TP_ERR_INVALID_ARG;
  if ((M > 0 && (!ptr_ok(X) || !ptr_ok(Y))) || !opt_ptr_ok(X) || !opt_ptr_ok(Y) || !shards_ok(W_shards, t))
    return TP_ERR_INVALID_ARG;
  if (K % t != 0 || (K / t) % 8 != 0 || N % 8 != 0) return TP_ERR_UNSUPPORTED_SHAPE;
  DeviceInfo* dev = nullptr;
  int st = device_ready(&dev);
  if (st != TP_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int kmaj = w_layout == TP_W_OUT_IN;
  if (dtype == TP_DTYPE_BF16)
    return run_gemm_tc(*dev, X, K, M, W_shards, t, 1, K / t, N, Y, N, out_dtype == TP_DTYPE_F32, TP_ACT_NONE, s, 1,
                       0, nullptr, kmaj);
  return run_gemm_simt(static_cast<const float*>(X), K, M, W_shards, t, 1, K / t, N, static_cast<float*>(Y), N,
                       TP_ACT_NONE, s, kmaj);
}

// -------------------------------------------- reduce + residual + LayerNorm
int tp_reduce_residual_layernorm(int S, int H, int nparts, const float* parts, const void* X, int x_dtype,
                                 const float* gamma, const float* beta, float eps, void* Y, int out_dtype,
                                 void* stream) {
  if (S < 0 || nparts < 0 || !valid_dtype(x_dtype) || !valid_dtype(out_dtype) || !(eps > 0.0f) ||
      !std::isfinite(eps))
    return TP_ERR_INVALID_ARG;
  if ((S > 0 && (!ptr_ok(X) || !ptr_ok(Y) || (nparts > 0 && !ptr_ok(parts)))) || !opt_ptr_ok(X) ||
      !opt_ptr_ok(Y) || !opt_ptr_ok(parts) || !opt_ptr_ok(gamma) || !opt_ptr_ok(beta))
    return TP_ERR_INVALID_ARG;
  if (!hidden_ok(H)) return TP_ERR_UNSUPPORTED_SHAPE;
  DeviceInfo* dev = nullptr;
  int st = device_ready(&dev);
  if (st != TP_OK) return st;
  return run_reduce_ln(S, H, nparts, parts, X, x_dtype == TP_DTYPE_BF16, gamma, beta, eps, Y,
                       out_dtype == TP_DTYPE_BF16, static_cast<cudaStream_t>(stream), dev->sm_count);
}

// ------------------------------------------------------------- GEMM tiling
int tp_reduce_residual_layernorm_multi(int rows, int H, int nparts, const float* const* parts, const void* X,
                                       int x_dtype, const float* gamma, const float* beta, float eps, int nout,
                                       void* const* Y_outs, int out_dtype, void* stream) {
  if (rows < 0 || nparts < 0 || nparts > TP_MAX_SHARDS || nout < 1 || nout > TP_MAX_SHARDS ||
      !valid_dtype(x_dtype) || !valid_dtype(out_dtype) || !(eps > 0.0f) || !std::isfinite(eps))
    return TP_ERR_INVALID_ARG;
  if ((nparts > 0 && !parts) || !Y_outs || !opt_ptr_ok(gamma) || !opt_ptr_ok(beta) || !opt_ptr_ok(X))
    return TP_ERR_INVALID_ARG;
  if (rows > 0) {
    if (!ptr_ok(X)) return TP_ERR_INVALID_ARG;
    for (int q = 0; q < nparts; ++q)
      if (!ptr_ok(parts[q])) return TP_ERR_INVALID_ARG;
    for (int o = 0; o < nout; ++o)
      if (!ptr_ok(Y_outs[o])) return TP_ERR_INVALID_ARG;
  }
  if (!hidden_ok(H)) return TP_ERR_UNSUPPORTED_SHAPE;
  DeviceInfo* dev = nullptr;
  int st = device_ready(&dev);
  if (st != TP_OK) return st;
  if (rows == 0) return TP_OK;
  return run_reduce_ln(rows, H, nparts, nullptr, X, x_dtype == TP_DTYPE_BF16, gamma, beta, eps, Y_outs[0],
                       out_dtype == TP_DTYPE_BF16, static_cast<cudaStream_t>(stream), dev->sm_count, 1, parts,
                       nout - 1, Y_outs + 1);
}

// ------------------------------------------------- one rank's partial sum
size_t tp_mlp_partial_workspace_bytes(int S, int H, int F, int t, int dtype) {
  if (S < 0 || H <= 0 || F <= 0 || t < 1 || !valid_dtype(dtype)) return 0;
  const size_t eh = dtype == TP_DTYPE_BF16 ? 2 : 4;
  return align256(static_cast<size_t>(S) * F * eh);
}

int tp_mlp_partial_forward(int S, int H, int F, int t, int dtype, const void* X, const void* const* A_shards,
                           const void* const* B_shards, int act, float* P, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (t < 1 || t > TP_MAX_SHARDS || S < 0 || H <= 0 || F <= 0 || !valid_dtype(dtype) || !valid_act(act))
    return TP_ERR_INVALID_ARG;
  if ((S > 0 && (!ptr_ok(X) || !ptr_ok(P))) || !opt_ptr_ok(X) || !opt_ptr_ok(P) || !shards_ok(A_shards, t) ||
      !shards_ok(B_shards, t) || !opt_ptr_ok(workspace))
    return TP_ERR_INVALID_ARG;
  if (F % t != 0 || (F / t) % 8 != 0 || H % 8 != 0) return TP_ERR_UNSUPPORTED_SHAPE;
  const size_t need = tp_mlp_partial_workspace_bytes(S, H, F, t, dtype);
  if (workspace_bytes < need || (need > 0 && !workspace)) return TP_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  int st = device_ready(&dev);
  if (st != TP_OK) return st;
  int nparts = 1;
  return mlp_products(*dev, S, H, F, t, dtype, X, A_shards, B_shards, act, workspace, P, 1, &nparts,
                      static_cast<cudaStream_t>(stream), 0);
}

size_t tp_attn_partial_workspace_bytes(int S, int H, int nh, int d, int t, int dtype) {
  if (S < 0 || H <= 0 || nh <= 0 || d <= 0 || t < 1 || dtype != TP_DTYPE_BF16) return 0;
  const size_t s = static_cast<size_t>(S), hl = static_cast<size_t>(nh) * d;
  return align256(s * 3 * hl * 2) + align256(s * hl * 2);
}

int tp_attn_partial_forward(int S, int H, int nh, int d, int t, int dtype, const void* X,
                            const void* const* Wqkv_shards, const void* const* Wo_shards, float* P, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (t < 1 || t > TP_MAX_SHARDS || S < 0 || H <= 0 || nh <= 0 || d <= 0 || dtype != TP_DTYPE_BF16)
    return TP_ERR_INVALID_ARG;
  if ((S > 0 && (!ptr_ok(X) || !ptr_ok(P))) || !opt_ptr_ok(X) || !opt_ptr_ok(P) || !shards_ok(Wqkv_shards, t) ||
      !shards_ok(Wo_shards, t) || !opt_ptr_ok(workspace))
    return TP_ERR_INVALID_ARG;
  if (d != tp::attn::D || nh % t != 0 || static_cast<long long>(nh) * d > H || H % 8 != 0 ||
      S % tp::attn::BQ != 0)
    return TP_ERR_UNSUPPORTED_SHAPE;
  const size_t need = tp_attn_partial_workspace_bytes(S, H, nh, d, t, dtype);
  if (workspace_bytes < need || (need > 0 && !workspace)) return TP_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  int st = device_ready(&dev);
  if (st != TP_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t hl = static_cast<size_t>(nh) * d;
  int nparts = 1;
  return attn_products(*dev, S, H, nh, d, t, X, Wqkv_shards, Wo_shards, ws, ws + align256(static_cast<size_t>(S) * 3 * hl * 2),
                       P, 1, &nparts, static_cast<cudaStream_t>(stream), 0, nullptr, nullptr, 0,
                       static_cast<size_t>(S) * H * 4);
}

// --------------------------------------------- peer access between ranks
// The handle is the CUDA IPC handle of the allocation that contains dev_ptr
// (a caching allocator hands out pieces of larger allocations) followed by
// dev_ptr's byte offset in it; an import maps the allocation and adds the
// offset.  Imports are remembered so that close can unmap by the address it
// returned.
static_assert(sizeof(cudaIpcMemHandle_t) + sizeof(unsigned long long) == TP_IPC_HANDLE_BYTES, "IPC handle size");
std::mutex g_ipc_mu;
struct IpcImport {
  void* addr;
  void* base;
};
IpcImport g_ipc_imports[1024];
int g_ipc_n = 0;

int tp_ipc_export(const void* dev_ptr, void* handle) {
  if (!dev_ptr || !handle) return TP_ERR_INVALID_ARG;
  static PFN_cuMemGetAddressRange_v3020 range_fn = nullptr;
  if (!range_fn) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return TP_ERR_CUDA;
    range_fn = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
  }
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range_fn(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS) return TP_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return TP_ERR_CUDA;
  const unsigned long long off = reinterpret_cast<CUdeviceptr>(dev_ptr) - base;
  std::memcpy(handle, &h, sizeof(h));
  std::memcpy(static_cast<uint8_t*>(handle) + sizeof(h), &off, sizeof(off));
  return TP_OK;
}

int tp_ipc_import(const void* handle, void** dev_ptr) {
  if (!handle || !dev_ptr) return TP_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  unsigned long long off = 0;
  std::memcpy(&h, handle, sizeof(h));
  std::memcpy(&off, static_cast<const uint8_t*>(handle) + sizeof(h), sizeof(off));
  std::lock_guard<std::mutex> lk(g_ipc_mu);
  if (g_ipc_n >= 1024) return TP_ERR_INVALID_ARG;
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return TP_ERR_CUDA;
  void* addr = static_cast<uint8_t*>(base) + off;
  g_ipc_imports[g_ipc_n++] = {addr, base};
  *dev_ptr = addr;
  return TP_OK;
}

int tp_ipc_close(void* dev_ptr) {
  if (!dev_ptr) return TP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_ipc_mu);
  for (int i = 0; i < g_ipc_n; ++i) {
    if (g_ipc_imports[i].addr == dev_ptr) {
      void* base = g_ipc_imports[i].base;
      g_ipc_imports[i] = g_ipc_imports[--g_ipc_n];
      return cudaIpcCloseMemHandle(base) == cudaSuccess ? TP_OK : TP_ERR_CUDA;
    }
  }
  return TP_ERR_INVALID_ARG;
}

int tp_peer_barrier(int nranks, int rank, unsigned long long* const* flags, unsigned long long epoch, void* stream) {
  if (nranks < 1 || nranks > TP_MAX_SHARDS || rank < 0 || rank >= nranks || !flags || epoch == 0)
    return TP_ERR_INVALID_ARG;
  for (int q = 0; q < nranks; ++q)
    if (!flags[q] || (reinterpret_cast<uintptr_t>(flags[q]) & 7u)) return TP_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  int st = device_ready(&dev);
  if (st != TP_OK) return st;
  tp::PeerBarrierArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int q = 0; q < nranks; ++q) a.flags[q] = flags[q];
  a.nranks = nranks;
  a.rank = rank;
  a.epoch = epoch;
  a.limit = tp::WAIT_LIMIT_CYCLES;
  tp::peer_barrier_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return launch_status();
}

int tp_set_gemm_tile_n(int tile_n) {
  if (tile_n != 0 && tile_n != 128 && (tile_n < 256 || tile_n > 512 || tile_n % 32 != 0))
    return TP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  g_force_tile_n = tile_n;
  return TP_OK;
}

int tp_set_gemm_stream_k(int mode) {
  if (mode < 0 || mode > 2) return TP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  g_stream_k = mode;
  return TP_OK;
}

int tp_gemm_plan_sk(int M, int t, int row_mode, int shard_k, int shard_n, int out_f32, int b_kmajor,
                    int heavy_epilogue, int slots, int max_splits, size_t sk_area_bytes, int* tile_n, int* splits,
                    int* stream_k, int* sk_clusters) {
  return tp_gemm_plan_ex(M, t, row_mode, shard_k, shard_n, out_f32, 0, b_kmajor, heavy_epilogue, slots, max_splits,
                         sk_area_bytes, tile_n, splits, stream_k, sk_clusters);
}

int tp_gemm_plan_ex(int M, int t, int row_mode, int shard_k, int shard_n, int out_f32, int a_mnmajor, int b_kmajor,
                    int heavy_epilogue, int slots, int max_splits, size_t sk_area_bytes, int* tile_n, int* splits,
                    int* stream_k, int* sk_clusters) {
  if (M < 1 || t < 1 || t > TP_MAX_SHARDS || shard_k < 1 || shard_n < 1 || slots < 1 || max_splits < 1 ||
      !tile_n || !splits)
    return TP_ERR_INVALID_ARG;
  tp::GemmArgs p;
  std::memset(&p, 0, sizeof(p));
  p.a_mnmajor = a_mnmajor ? 1 : 0;
  p.M = M;
  p.t = t;
  p.row_mode = row_mode ? 1 : 0;
  p.shard_k = shard_k;
  p.shard_n = shard_n;
  p.k_blocks = ceil_div(shard_k, tp::GemmCfg<1>::BK) * (row_mode ? t : 1);
  p.out_f32 = out_f32 ? 1 : 0;
  p.b_kmajor = b_kmajor ? 1 : 0;
  p.epi_mode = heavy_epilogue ? tp::EPI_GRAD : tp::EPI_PLAIN;
  const TilePlan plan = plan_tiles(p, M >= TP_GEMM_PAIR_MIN_ROWS, slots, out_f32 ? max_splits : 1, sk_area_bytes);
  *tile_n = plan.tile_n;
  *splits = plan.splits;
  if (stream_k) *stream_k = plan.stream_k;
  if (sk_clusters) *sk_clusters = plan.sk_clusters;
  return TP_OK;
}

int tp_gemm_plan(int M, int t, int row_mode, int shard_k, int shard_n, int out_f32, int b_kmajor,
                 int heavy_epilogue, int slots, int max_splits, int* tile_n, int* splits) {
  return tp_gemm_plan_sk(M, t, row_mode, shard_k, shard_n, out_f32, b_kmajor, heavy_epilogue, slots, max_splits, 0,
                         tile_n, splits, nullptr, nullptr);
}

int tp_set_attn_kv_split(int mode) {
  if (mode < 0 || mode > 2) return TP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  g_attn_split = mode;
  return TP_OK;
}

int tp_attn_split_plan(int S, int nh, int slots, int mode, size_t scratch_bytes, int* whole, int* split,
                       int* kv_half) {
  if (S < 0 || nh < 1 || slots < 1 || mode < 0 || mode > 2 || !whole || !split || !kv_half) return TP_ERR_INVALID_ARG;
  const AttnSplit p = attn_split_plan(S, nh, slots, mode, scratch_bytes);
  *whole = p.whole;
  *split = p.split;
  *kv_half = p.kv_half;
  return TP_OK;
}

// ------------------------------------------------------------- self-test
int tp_selftest_flag_wait_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles < 1) return TP_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  int st = device_ready(&dev);
  if (st != TP_OK) return st;
  tp::selftest_flag_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles);
  return launch_status();
}

int tp_selftest_exp2(const float* x, float* y_poly, float* y_exp2f, int n, void* stream) {
  return tp_selftest_exp2_form(x, y_poly, y_exp2f, n, 0, stream);
}

int tp_selftest_exp2_form(const float* x, float* y_poly, float* y_exp2f, int n, int form, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y_poly || !y_exp2f)) || form < 0 || form > 1) return TP_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  int st = device_ready(&dev);
  if (st != TP_OK) return st;
  if (n == 0) return TP_OK;
  const int blocks = ceil_div(n, 256) < 4 * dev->sm_count ? ceil_div(n, 256) : 4 * dev->sm_count;
  tp::selftest_exp2_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_exp2f, n, form);
  return launch_status();
}

int tp_selftest_wait_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles < 1) return TP_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  int st = device_ready(&dev);
  if (st != TP_OK) return st;
  tp::selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles);
  return launch_status();
}

// ------------------------------------------------------------- profiling
int tp_profile_enable(int on) {
  if (on && !g_prof_events_made) {
    for (int i = 0; i < PROF_CAP; ++i) {
      if (cudaEventCreate(&g_ev_start[i]) != cudaSuccess || cudaEventCreate(&g_ev_stop[i]) != cudaSuccess)
        return TP_ERR_CUDA;
    }
    g_prof_events_made = true;
  }
  g_prof_on = on != 0;
  g_prof_sampling = true;
  g_prof_n = 0;
  for (int k = 0; k < PROF_KINDS; ++k) g_prof_launches[k] = 0;
  return TP_OK;
}

int tp_profile_sample(int on) {
  g_prof_sampling = on != 0;
  return TP_OK;
}

int tp_profile_collect(int* launches, int* timed, double* ms, int max_kinds) {
  const int nk = max_kinds < PROF_KINDS ? max_kinds : PROF_KINDS;
  for (int k = 0; k < nk; ++k) {
    if (launches) launches[k] = static_cast<int>(g_prof_launches[k]);
    if (timed) timed[k] = 0;
    if (ms) ms[k] = 0.0;
  }
  for (int i = 0; i < g_prof_n; ++i) {
    const int k = g_prof_kind[i];
    if (k >= nk) continue;
    float t = 0.0f;
    if (cudaEventSynchronize(g_ev_stop[i]) != cudaSuccess ||
        cudaEventElapsedTime(&t, g_ev_start[i], g_ev_stop[i]) != cudaSuccess)
      return -TP_ERR_CUDA;
    if (timed) timed[k] += 1;
    if (ms) ms[k] += t;
  }
  g_prof_n = 0;
  for (int k = 0; k < PROF_KINDS; ++k) g_prof_launches[k] = 0;
  return nk;
}

const char* tp_kernel_kind_name(int kind) {
  switch (kind) {
    case K_GEMM_TC: return "gemm_tcgen05";
    case K_REDUCE_LN: return "reduce_residual_layernorm";
    case K_GEMM_SIMT: return "gemm_simt_f32";
    case K_ATTN: return "attention_fwd";
    case K_LN_BACK: return "layernorm_backward";
    case K_ATTN_BACK: return "attention_backward_elementwise";
    case K_LN_PARAMS: return "layernorm_grad_params";
    case K_ATTN_BWD: return "attention_bwd";
    default: return "unknown";
  }
}

}  // extern "C"
