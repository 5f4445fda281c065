// Combine kernel: one warp per token (combine.cuh holds the per-token gather-sum and its
// source).
#include "combine.cuh"
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) combine_kernel(const void* __restrict__ y, int y_f32,
                                                      const int32_t* __restrict__ slot_of,
                                                      const float* __restrict__ topk_w, int T,
                                                      int k, int H, void* __restrict__ out,
                                                      int out_f32) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  combine_token(y, y_f32, slot_of, topk_w, t, k, H, out, out_f32, threadIdx.x & 31);
}

}  // namespace

cudaError_t launch_combine(const void* y, int y_f32, const int32_t* slot_of, const float* topk_w,
                           int T, int k, int H, void* out, int out_f32, cudaStream_t s) {
  const int warps = 8;
  count_launch();
  combine_kernel<<<(T + warps - 1) / warps, 32 * warps, 0, s>>>(y, y_f32, slot_of, topk_w, T, k,
                                                                H, out, out_f32);
  return cudaGetLastError();
}

}  // namespace moe
