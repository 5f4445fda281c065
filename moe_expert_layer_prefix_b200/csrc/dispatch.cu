// Dispatch kernels (dispatch.cuh holds the per-chunk steps, their ordering rule and their
// source): hist -> scan -> offsets -> slots -> row copies.
#include "common.cuh"
#include "dispatch.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kWarps = 8;  // chunks per block in hist / scatter

__global__ void __launch_bounds__(32 * kWarps) hist_kernel(const int32_t* __restrict__ topk_idx,
                                                           int T, int E, int k, int C,
                                                           int32_t* __restrict__ cnt) {
  extern __shared__ uint32_t smask[];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * kWarps + w;
  if (chunk >= C) return;
  hist_chunk(smask + w * E, topk_idx, T, E, k, chunk, lane, cnt);
}

__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ cnt, int E, int C,
                                                    int32_t* __restrict__ totals) {
  __shared__ int32_t part[32][33];
  scan_group(cnt, E, C, totals, blockIdx.x, 32, threadIdx.x >> 5, threadIdx.x & 31, part);
}

__global__ void __launch_bounds__(1024) offsets_kernel(const int32_t* __restrict__ totals, int E,
                                                       int32_t* __restrict__ offsets) {
  __shared__ int32_t wsum[32];
  offsets_from_totals(totals, E, offsets, wsum);
}

__global__ void __launch_bounds__(32 * kWarps) slots_kernel(
    const int32_t* __restrict__ topk_idx, int T, int E, int k, int C,
    const int32_t* __restrict__ bases, const int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm_src, int32_t* __restrict__ slot_of) {
  extern __shared__ uint32_t smask[];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * kWarps + w;
  if (chunk >= C) return;
  assign_slots_chunk(smask + w * E, topk_idx, T, E, k, chunk, bases, offsets, perm_src, slot_of,
                     lane);
}

__global__ void __launch_bounds__(256) copy_rows_kernel(
    const uint8_t* __restrict__ x, const float* __restrict__ x_scales, int row_bytes, int nscale,
    const int32_t* __restrict__ slot_of, int T, int k, uint8_t* __restrict__ x_perm,
    float* __restrict__ x_perm_scales) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  copy_token_rows(x, x_scales, row_bytes, nscale, slot_of, t, k, x_perm, x_perm_scales,
                  threadIdx.x & 31);
}

// One warp per token: BF16 row -> E4M3 codes + 1x128 scales in each of its k slots.
__global__ void __launch_bounds__(256) quant_copy_rows_kernel(
    const __nv_bfloat16* __restrict__ x, int H, const int32_t* __restrict__ slot_of, int T,
    int k, uint8_t* __restrict__ x_perm, float* __restrict__ x_perm_scales) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  quant_copy_token_rows(x, H, slot_of, t, k, x_perm, x_perm_scales, threadIdx.x & 31);
}

}  // namespace

cudaError_t launch_dispatch(const void* x, const float* x_scales, int row_bytes, int T, int H,
                            int E, int k, const int32_t* topk_idx, void* x_perm,
                            float* x_perm_scales, int32_t* offsets, int32_t* perm_src,
                            int32_t* slot_of, void* ws, cudaStream_t s, bool quantize) {
  const int C = (T + kChunkTokens - 1) / kChunkTokens;
  int32_t* cnt = static_cast<int32_t*>(ws);
  const size_t cnt_bytes = ((static_cast<size_t>(C) * E * 4 + 255) / 256) * 256;
  int32_t* totals = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + cnt_bytes);
  const int blocks = (C + kWarps - 1) / kWarps;
  const size_t smem = static_cast<size_t>(kWarps) * E * 4;
  // the scatter kernel also holds a static slot table; opt in to the full size every time
  cudaError_t err = cudaFuncSetAttribute(hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(slots_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  count_launch(5);
  hist_kernel<<<blocks, 32 * kWarps, smem, s>>>(topk_idx, T, E, k, C, cnt);
  scan_kernel<<<(E + 31) / 32, 1024, 0, s>>>(cnt, E, C, totals);
  offsets_kernel<<<1, 1024, 0, s>>>(totals, E, offsets);
  slots_kernel<<<blocks, 32 * kWarps, smem, s>>>(topk_idx, T, E, k, C, cnt, offsets, perm_src,
                                                 slot_of);
  if (quantize)
    quant_copy_rows_kernel<<<(T + 7) / 8, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), H,
                                                     slot_of, T, k, static_cast<uint8_t*>(x_perm),
                                                     x_perm_scales);
  else
    copy_rows_kernel<<<(T + 7) / 8, 256, 0, s>>>(static_cast<const uint8_t*>(x), x_scales,
                                                 row_bytes, H / 128, slot_of, T, k,
                                                 static_cast<uint8_t*>(x_perm), x_perm_scales);
  return cudaGetLastError();
}

}  // namespace moe
