// Router kernel: one warp per token (route.cuh holds the per-token selection, its scoring
// rules and their source).
#include "common.cuh"
#include "internal.h"
#include "route.cuh"

namespace moe {
namespace {

template <int NPL>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits,
                                                    const float* __restrict__ bias, int T, int E,
                                                    int k, int sigmoid, int renorm,
                                                    int32_t* __restrict__ topk_idx,
                                                    float* __restrict__ topk_w) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  route_token<NPL>(logits, bias, t, E, k, sigmoid, renorm, topk_idx, topk_w, threadIdx.x & 31);
}

}  // namespace

cudaError_t launch_route(const float* logits, const float* bias, int T, int E, int k, int score,
                         int renorm, int32_t* topk_idx, float* topk_w, cudaStream_t s) {
  const int warps = 8;
  dim3 grid((T + warps - 1) / warps), block(32 * warps);
  const int sig = score == MOE_SCORE_SIGMOID;
  const int npl = (E + 31) / 32;
  count_launch();
  if (npl <= 1)
    route_kernel<1><<<grid, block, 0, s>>>(logits, bias, T, E, k, sig, renorm, topk_idx, topk_w);
  else if (npl <= 2)
    route_kernel<2><<<grid, block, 0, s>>>(logits, bias, T, E, k, sig, renorm, topk_idx, topk_w);
  else if (npl <= 4)
    route_kernel<4><<<grid, block, 0, s>>>(logits, bias, T, E, k, sig, renorm, topk_idx, topk_w);
  else if (npl <= 8)
    route_kernel<8><<<grid, block, 0, s>>>(logits, bias, T, E, k, sig, renorm, topk_idx, topk_w);
  else if (npl <= 16)
    route_kernel<16><<<grid, block, 0, s>>>(logits, bias, T, E, k, sig, renorm, topk_idx, topk_w);
  else
    route_kernel<32><<<grid, block, 0, s>>>(logits, bias, T, E, k, sig, renorm, topk_idx, topk_w);
  return cudaGetLastError();
}

}  // namespace moe
