// moe_dispatch_noalloc: the dispatch step for callers that cannot allocate device memory.
//
// moe_dispatch needs a caller-provided scratch workspace (per-chunk expert counts and the
// expert totals).  Some callers have no way to provide one: a host that owns no device
// allocator of its own (plain C code driving the library directly), a serving runtime that
// plans every device byte at start-up and forbids allocations afterwards, or a latency path
// that must not call cudaMalloc / cudaFree because those calls can synchronise the device.
// This entry point runs the same dispatch kernels with their scratch taken from a fixed
// buffer compiled into the library instead.
//
// The buffer is a file-scope __device__ array, so every GPU that loads the library holds
// it (kNoAllocScratchBytes) until the process exits.  Host code cannot use the array's name
// as a device address; the first call on each device looks the address up with
// cudaGetSymbolAddress while that device is current and caches it.
//
// All calls on a device share the one buffer.  Dispatch overwrites every scratch word it
// later reads, so nothing needs clearing between calls, but calls whose executions overlap
// on the GPU (different streams, or different host threads) race on the buffer and must
// be serialised by the caller.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB per device

static __device__ __align__(256) unsigned char g_dispatch_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_dispatch_scratch on the current device (looked up once per device).
moe_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_dispatch_noalloc(const void* x, const float* x_scales, int act, int T,
                                           int H, int E, int k, const int32_t* topk_idx,
                                           void* x_perm, float* x_perm_scales,
                                           int32_t* expert_offsets, int32_t* perm_src,
                                           int32_t* slot_of, cudaStream_t stream) {
  if (T < 1 || E < 1 || E > 1024) return MOE_ERR_INVALID_ARG;
  if (moe::dispatch_ws_bytes(T, E) > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
  void* scratch = nullptr;
  const moe_status st = scratch_address(&scratch);
  if (st != MOE_OK) return st;
  return moe_dispatch(x, x_scales, act, T, H, E, k, topk_idx, x_perm, x_perm_scales,
                      expert_offsets, perm_src, slot_of, scratch, kNoAllocScratchBytes, stream);
}
