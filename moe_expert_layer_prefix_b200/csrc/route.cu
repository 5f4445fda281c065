// Router kernel: one warp per token (route.cuh holds the per-token selection, its scoring
// rules and their source).
#include "common.cuh"
#include "internal.h"
#include "route.cuh"

namespace moe {
namespace {

constexpr int kRouteWarps = 8;

template <int NPL>
__global__ void __launch_bounds__(32 * kRouteWarps, 3) route_kernel(const float* __restrict__ logits,
                                                    const float* __restrict__ bias, int T, int E,
                                                    int k, int sigmoid, int renorm,
                                                    int32_t* __restrict__ topk_idx,
                                                    float* __restrict__ topk_w, int n_group,
                                                    int topk_group, float scale) {
  __shared__ __align__(8) uint8_t scratch[kRouteWarps][kRouteScratchBytes];
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  route_token<NPL>(logits, bias, t, E, k, sigmoid, renorm, topk_idx, topk_w, threadIdx.x & 31,
                   scratch[threadIdx.x >> 5], n_group, topk_group, scale);
}

}  // namespace

cudaError_t launch_route(const float* logits, const float* bias, int T, int E, int k, int score,
                         int renorm, int32_t* topk_idx, float* topk_w, cudaStream_t s,
                         int n_group, int topk_group, float scale) {
  dim3 grid((T + kRouteWarps - 1) / kRouteWarps), block(32 * kRouteWarps);
  const int sig = score == MOE_SCORE_SIGMOID;
  const int npl = (E + 31) / 32;
  count_launch();
#define MOE_ROUTE(N)                                                                        \
  route_kernel<N><<<grid, block, 0, s>>>(logits, bias, T, E, k, sig, renorm, topk_idx, topk_w, \
                                         n_group, topk_group, scale)
  if (npl <= 1) MOE_ROUTE(1);
  else if (npl <= 2) MOE_ROUTE(2);
  else if (npl <= 4) MOE_ROUTE(4);
  else if (npl <= 8) MOE_ROUTE(8);
  else if (npl <= 16) MOE_ROUTE(16);
  else MOE_ROUTE(32);
#undef MOE_ROUTE
  return cudaGetLastError();
}

}  // namespace moe
