// Combine kernel: one warp per (token, column chunk) (combine.cuh holds the gather-sum and its
// source).
#include "combine.cuh"
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// One warp per (token, column chunk); nc chunks per token (1: the whole row).
template <bool kF32, int kV>
__global__ void __launch_bounds__(256) combine_kernel(const void* __restrict__ y,
                                                      const int32_t* __restrict__ slot_of,
                                                      const float* __restrict__ topk_w, int T,
                                                      int k, int H, void* __restrict__ out,
                                                      int nc) {
  const long item = static_cast<long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (item >= static_cast<long>(T) * nc) return;
  const int t = static_cast<int>(item / nc), c = static_cast<int>(item % nc);
  const int width = nc == 1 ? H / 8 : 32 * kV;
  combine_token<kF32, kV>(y, slot_of, topk_w, t, k, H, out, threadIdx.x & 31, c * width,
                          (c + 1) * width);
}

// Mixed formats (BF16 y into fp32 out or the reverse) take this simple path.
__global__ void __launch_bounds__(256) combine_mixed_kernel(const void* __restrict__ y, int y_f32,
                                                            const int32_t* __restrict__ slot_of,
                                                            const float* __restrict__ topk_w,
                                                            int T, int k, int H,
                                                            void* __restrict__ out, int out_f32) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  for (int c = lane; c < H; c += 32) {
    float acc = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int slot = __ldcg(slot_of + static_cast<size_t>(t) * k + j);
      const float w = __ldcg(topk_w + static_cast<size_t>(t) * k + j);
      const size_t i = static_cast<size_t>(slot) * H + c;
      const float v = y_f32 ? __ldcg(static_cast<const float*>(y) + i)
                            : __bfloat162float(static_cast<const __nv_bfloat16*>(y)[i]);
      acc = fmaf(w, v, acc);
    }
    const size_t o = static_cast<size_t>(t) * H + c;
    if (out_f32) static_cast<float*>(out)[o] = acc;
    else static_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(acc);
  }
}

}  // namespace

cudaError_t launch_combine(const void* y, int y_f32, const int32_t* slot_of, const float* topk_w,
                           int T, int k, int H, void* out, int out_f32, cudaStream_t s) {
  const int warps = 8;
  count_launch();
  // one warp per 512 columns of a token with two 16-byte loads per lane and source row in
  // flight per pass: the fastest of the shapes measured on the V3, skewed and decode layers
  const int nc = combine_chunks<2>(H);
  const long items = static_cast<long>(T) * nc;
  const dim3 block(32 * warps);
  const dim3 grid(y_f32 == out_f32 ? static_cast<unsigned>((items + warps - 1) / warps)
                                   : static_cast<unsigned>((T + warps - 1) / warps));
  if (y_f32 && out_f32)
    combine_kernel<true, 2><<<grid, block, 0, s>>>(y, slot_of, topk_w, T, k, H, out, nc);
  else if (!y_f32 && !out_f32)
    combine_kernel<false, 2><<<grid, block, 0, s>>>(y, slot_of, topk_w, T, k, H, out, nc);
  else
    combine_mixed_kernel<<<grid, block, 0, s>>>(y, y_f32, slot_of, topk_w, T, k, H, out, out_f32);
  return cudaGetLastError();
}

}  // namespace moe
