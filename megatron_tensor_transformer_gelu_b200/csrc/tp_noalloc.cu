// tp_mlp_forward_noalloc: the MLP sublayer with its scratch in a fixed device
// array owned by this library, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc, for example:
//  * plugin hosts that give each plugin a fixed memory budget and forbid
//    allocation inside the plugin's execute hook;
//  * latency-critical loops, where cudaMalloc's implicit device-wide
//    synchronisation would stall every other stream;
//  * programs whose own caching allocator has reserved the device memory, so
//    an allocation from a library would fail or fragment that pool.
// Such callers pass inputs and outputs only; the scratch lives in
// g_tp_noalloc_scratch below.
//
// Costs and limits:
//  * Every GPU that loads this library holds TP_NOALLOC_SCRATCH_BYTES of
//    device memory for the array until the process exits.
//  * The array is shared by every call on a device and keeps the last call's
//    contents.  Calls whose kernels overlap on the GPU (different streams,
//    no ordering between them) race on it.  The sublayer overwrites every
//    scratch byte it reads before reading it, so nothing needs clearing.
//  * In host code `g_tp_noalloc_scratch` names a host-side stand-in, not a
//    device address.  Its device address is looked up once per device with
//    cudaGetSymbolAddress, with that device current, during the first call
//    on that device whose arguments pass the checks (an empty call with
//    S == 0 is enough).  Make that first call before any stream capture.
//  * Order of checks: the arguments (as tp_mlp_forward checks them), then
//    the address lookup, then the size limit.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/tpblock.h"
#include "tp_internal.h"

namespace {

// The largest workspace a no-alloc call may need (tp_mlp_workspace_bytes).
constexpr size_t TP_NOALLOC_SCRATCH_BYTES = size_t(32) << 20;  // 32 MiB

static __device__ __align__(256) unsigned char g_tp_noalloc_scratch[TP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (resolved once).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TP_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_tp_noalloc_scratch) != cudaSuccess || p == nullptr) return TP_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return TP_OK;
}

}  // namespace

extern "C" {

size_t tp_noalloc_scratch_bytes(void) { return TP_NOALLOC_SCRATCH_BYTES; }

int tp_mlp_forward_noalloc(int S, int H, int F, int t, int dtype, int out_dtype, const void* X,
                           const void* const* A_shards, const void* const* B_shards, const float* gamma,
                           const float* beta, float eps, int act, void* Y, void* stream) {
  // 1. The same argument checks as tp_mlp_forward, in the same order.
  int st = tp_internal_check_mlp_args(S, H, F, t, dtype, out_dtype, X, A_shards, B_shards, gamma, beta, eps, act, Y);
  if (st != TP_OK) return st;
  // 2. The scratch array's device address on the current device, looked up on
  //    the first call there (an empty call, S == 0, does it too).
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != TP_OK) return st;
  // 3. The size limit: nothing is launched for sizes the array cannot hold.
  if (tp_mlp_workspace_bytes(S, H, F, t, dtype) > TP_NOALLOC_SCRATCH_BYTES) return TP_ERR_WORKSPACE_TOO_SMALL;
  return tp_mlp_forward(S, H, F, t, dtype, out_dtype, X, A_shards, B_shards, gamma, beta, eps, act, Y, scratch,
                        TP_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
