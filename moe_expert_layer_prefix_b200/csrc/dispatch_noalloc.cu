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
// as a device address: every call looks the address up with cudaGetSymbolAddress while
// the caller's device is current (the lookup is cheap, and nothing is cached, so a reset
// device or a new context never sees a stale address).  The first call on a device also
// loads the library's module there; make it before any stream capture.
//
// All calls on a device share the one buffer.  Dispatch overwrites every scratch word it
// later reads, so nothing needs clearing between calls, but calls whose executions overlap
// on the GPU (different streams, or different host threads) race on the buffer and must
// be serialised by the caller.
#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB per device

static __device__ __align__(256) unsigned char g_dispatch_scratch[kNoAllocScratchBytes];

}  // namespace

extern "C" moe_status moe_dispatch_noalloc(const void* x, const float* x_scales, int act, int T,
                                           int H, int E, int k, const int32_t* topk_idx,
                                           void* x_perm, float* x_perm_scales,
                                           int32_t* expert_offsets, int32_t* perm_src,
                                           int32_t* slot_of, cudaStream_t stream) {
  // the shape checks of moe_dispatch come first, so both entry points give the same status
  // for a shape neither supports; only then is the buffer's size the deciding limit
  const moe_status shapes = moe::check_dispatch_shapes(T, H, E, k);
  if (shapes != MOE_OK) return shapes;
  if (moe::dispatch_ws_bytes(T, E) > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (cudaGetSymbolAddress(&scratch, g_dispatch_scratch) != cudaSuccess || scratch == nullptr)
    return MOE_ERR_CUDA;
  return moe_dispatch(x, x_scales, act, T, H, E, k, topk_idx, x_perm, x_perm_scales,
                      expert_offsets, perm_src, slot_of, scratch, kNoAllocScratchBytes, stream);
}
