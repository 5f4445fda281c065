// Self-test of the library's bounded waits: kernels whose waits can never be satisfied, by
// construction, so that a test can watch each wait give up, record MOE_ERR_TIMEOUT with its
// site in the device error word and return, leaving the context usable.  Nothing here
// traps, faults or spins without a limit.  (The source pages have no counterpart; this
// checks the library's own failure detection.)
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// grid-barrier words of the self-test (zeroed before each launch)
static __device__ uint32_t g_selftest_bar[2];

__global__ void __launch_bounds__(32, 1) wait_selftest_kernel(int kind, uint32_t* bar, int* err) {
  if (kind == MOE_SELFTEST_MBARRIER) {
    // one CTA: an mbarrier expecting one arrival that nothing makes
    if (blockIdx.x != 0) return;
    __shared__ __align__(8) uint64_t mbar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
      mbar_init(&mbar, 1);
      abort = 0;
      fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&mbar, 0, err, SITE_SELFTEST_MBAR, &abort);
    __syncthreads();
  } else {
    // every CTA arrives at a grid barrier that expects one arrival more than the grid has
    grid_sync(bar, err, gridDim.x + 1);
  }
}

}  // namespace

cudaError_t launch_wait_selftest(int kind, int* err, cudaStream_t s) {
  void* bar = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&bar, g_selftest_bar);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(bar, 0, 2 * sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kind == MOE_SELFTEST_MBARRIER ? 1 : num_sms());
  cfg.blockDim = dim3(32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, wait_selftest_kernel, kind, static_cast<uint32_t*>(bar), err);
}

}  // namespace moe

extern "C" moe_status moe_selftest_wait(int kind, cudaStream_t stream) {
  if (kind != MOE_SELFTEST_MBARRIER && kind != MOE_SELFTEST_GRID_BARRIER)
    return MOE_ERR_INVALID_ARG;
  int* err = moe::device_error_word();
  if (err == nullptr) return MOE_ERR_CUDA;
  return moe::launch_wait_selftest(kind, err, stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
