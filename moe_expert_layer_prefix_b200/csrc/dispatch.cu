// Dispatch: stable counting sort of the T*k (token, rank) pairs by expert, and the row
// copies x -> x_perm.
//
// The pages' pipeline starts by dispatching tokens to their experts (jiqizhixin,
// "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了", section "Mega MoE 是什么？", pipeline
// paragraph) through a token-to-expert mapping with a fused expand (youleyou, "DeepSeek
// 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", Tile Kernels feature list, routing item).
// Order inside an expert is ascending token id, which makes the result unique and lets
// every step be deterministic without atomics on the data path:
//
//   tokens are cut into 32-token chunks; in a chunk, the set of tokens that chose expert e
//   is a 32-bit mask built with shared-memory atomicOr (order independent).
//   slot(t, j) = offsets[e] + (tokens of e in earlier chunks) + popc(mask_e & below(t)).
//
// Kernels: hist (per-chunk counts) -> scan (per-expert exclusive scan over chunks, totals)
// -> offsets (exclusive scan over experts) -> scatter (slots, permutation, row copies).
// The row copy reads each x row once and writes it k times with 16-byte accesses.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kWarps = 8;  // chunks per block in hist / scatter

// Builds, in smem, mask[e] for the warp's chunk.  `mask` has E words for this warp.
__device__ __forceinline__ void build_chunk_mask(uint32_t* mask, const int32_t* topk_idx, int T,
                                                 int E, int k, int chunk, int lane) {
  for (int e = lane; e < E; e += 32) mask[e] = 0u;
  __syncwarp();
  const int t = chunk * kChunkTokens + lane;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = __ldg(topk_idx + static_cast<size_t>(t) * k + j);
      atomicOr(mask + e, 1u << lane);
    }
  }
  __syncwarp();
}

__global__ void __launch_bounds__(32 * kWarps) hist_kernel(const int32_t* __restrict__ topk_idx,
                                                           int T, int E, int k, int C,
                                                           int32_t* __restrict__ cnt) {
  extern __shared__ uint32_t smask[];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * kWarps + w;
  if (chunk >= C) return;
  uint32_t* mask = smask + w * E;
  build_chunk_mask(mask, topk_idx, T, E, k, chunk, lane);
  for (int e = lane; e < E; e += 32) cnt[static_cast<size_t>(chunk) * E + e] = __popc(mask[e]);
}

// Per expert, exclusive scan of the chunk counts (in place: cnt becomes the chunk bases) and
// the expert totals.  Block: 32 experts (lanes) x 32 warps, warp w owns a range of chunks.
__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ cnt, int E, int C,
                                                    int32_t* __restrict__ totals) {
  __shared__ int32_t part[32][33];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 32 + lane;
  const int per = (C + 31) / 32;
  const int c0 = w * per, c1 = min(C, c0 + per);
  int sum = 0;
  if (e < E)
    for (int c = c0; c < c1; ++c) sum += cnt[static_cast<size_t>(c) * E + e];
  part[w][lane] = sum;
  __syncthreads();
  if (w == 0) {
    int run = 0;
    for (int i = 0; i < 32; ++i) {
      const int v = part[i][lane];
      part[i][lane] = run;
      run += v;
    }
    if (e < E) totals[e] = run;
  }
  __syncthreads();
  int run = part[w][lane];
  if (e < E)
    for (int c = c0; c < c1; ++c) {
      int32_t* p = cnt + static_cast<size_t>(c) * E + e;
      const int v = *p;
      *p = run;
      run += v;
    }
}

// expert_offsets[0..E] = exclusive scan of totals (E <= 1024, one block).
__global__ void __launch_bounds__(1024) offsets_kernel(const int32_t* __restrict__ totals, int E,
                                                       int32_t* __restrict__ offsets) {
  __shared__ int32_t wsum[32];
  const int i = threadIdx.x, lane = i & 31, w = i >> 5;
  const int v = (i < E) ? totals[i] : 0;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) wsum[w] = incl;
  __syncthreads();
  if (w == 0) {
    int s = wsum[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += o;
    }
    wsum[lane] = s;  // inclusive
  }
  __syncthreads();
  const int base = (w == 0) ? 0 : wsum[w - 1];
  if (i < E) offsets[i] = base + incl - v;
  if (i == E - 1) offsets[E] = base + incl;
}

__global__ void __launch_bounds__(32 * kWarps) scatter_kernel(
    const uint8_t* __restrict__ x, const float* __restrict__ x_scales, int row_bytes, int nscale,
    const int32_t* __restrict__ topk_idx, int T, int E, int k, int C,
    const int32_t* __restrict__ bases, const int32_t* __restrict__ offsets,
    uint8_t* __restrict__ x_perm, float* __restrict__ x_perm_scales,
    int32_t* __restrict__ perm_src, int32_t* __restrict__ slot_of) {
  extern __shared__ uint32_t smask[];
  __shared__ int32_t sslot[kWarps][kChunkTokens][32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * kWarps + w;
  if (chunk >= C) return;
  uint32_t* mask = smask + w * E;
  build_chunk_mask(mask, topk_idx, T, E, k, chunk, lane);

  const int t = chunk * kChunkTokens + lane;
  if (t < T) {
    const uint32_t below = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = __ldg(topk_idx + static_cast<size_t>(t) * k + j);
      const int slot = __ldg(offsets + e) + __ldg(bases + static_cast<size_t>(chunk) * E + e) +
                       __popc(mask[e] & below);
      const int src = t * k + j;
      slot_of[src] = slot;
      perm_src[slot] = src;
      sslot[w][lane][j] = slot;
    }
  }
  __syncwarp();

  // row copies: the warp walks its chunk's tokens; each 16-byte piece of a row is loaded
  // once and stored to the token's k slots
  const int ntok = min(kChunkTokens, T - chunk * kChunkTokens);
  const int nvec = row_bytes / 16;
  for (int i = 0; i < ntok; ++i) {
    const int tt = chunk * kChunkTokens + i;
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(tt) * row_bytes);
    for (int v = lane; v < nvec; v += 32) {
      const uint4 d = __ldg(src + v);
      for (int j = 0; j < k; ++j) {
        uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(sslot[w][i][j]) *
                                                           row_bytes);
        dst[v] = d;
      }
    }
    if (x_scales != nullptr) {
      for (int v = lane; v < nscale; v += 32) {
        const float sv = __ldg(x_scales + static_cast<size_t>(tt) * nscale + v);
        for (int j = 0; j < k; ++j)
          x_perm_scales[static_cast<size_t>(sslot[w][i][j]) * nscale + v] = sv;
      }
    }
  }
}

}  // namespace

cudaError_t launch_dispatch(const void* x, const float* x_scales, int row_bytes, int T, int H,
                            int E, int k, const int32_t* topk_idx, void* x_perm,
                            float* x_perm_scales, int32_t* offsets, int32_t* perm_src,
                            int32_t* slot_of, void* ws, cudaStream_t s) {
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
  err = cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  count_launch(4);
  hist_kernel<<<blocks, 32 * kWarps, smem, s>>>(topk_idx, T, E, k, C, cnt);
  scan_kernel<<<(E + 31) / 32, 1024, 0, s>>>(cnt, E, C, totals);
  offsets_kernel<<<1, 1024, 0, s>>>(totals, E, offsets);
  scatter_kernel<<<blocks, 32 * kWarps, smem, s>>>(
      static_cast<const uint8_t*>(x), x_scales, row_bytes, H / 128, topk_idx, T, E, k, C, cnt,
      offsets, static_cast<uint8_t*>(x_perm), x_perm_scales, perm_src, slot_of);
  return cudaGetLastError();
}

}  // namespace moe
