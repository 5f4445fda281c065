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
// Steps: hist (per-chunk counts) -> scan (per-expert exclusive scan over chunks, totals)
// -> offsets (exclusive scan over experts) -> slots (permutation) -> row copies (one warp
// per token, each x row read once and written k times with 16-byte accesses).
// These device functions are shared by the dispatch kernels and the persistent forward
// kernel.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {

// Data that the persistent forward kernel produces in an earlier phase (routing indices,
// counts, totals) is read with ld.global.cg, never through the non-coherent path.

// Builds, in shared memory, mask[e] for one 32-token chunk: bit i is set if token
// chunk*32 + i selected expert e.  `mask` holds E words for this warp.
__device__ __forceinline__ void build_chunk_mask(uint32_t* mask, const int32_t* topk_idx, int T,
                                                 int E, int k, int chunk, int lane) {
  for (int e = lane; e < E; e += 32) mask[e] = 0u;
  __syncwarp();
  const int t = chunk * kChunkTokens + lane;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = __ldcg(topk_idx + static_cast<size_t>(t) * k + j);
      atomicOr(mask + e, 1u << lane);
    }
  }
  __syncwarp();
}

// cnt[chunk][e] = number of tokens of the chunk that selected e (one warp).
__device__ __forceinline__ void hist_chunk(uint32_t* mask, const int32_t* topk_idx, int T, int E,
                                           int k, int chunk, int lane, int32_t* cnt) {
  build_chunk_mask(mask, topk_idx, T, E, k, chunk, lane);
  for (int e = lane; e < E; e += 32) cnt[static_cast<size_t>(chunk) * E + e] = __popc(mask[e]);
}

// For the 32 experts [32g, 32g + 32): exclusive scan of cnt[.][e] over the C chunks, in place
// (cnt becomes the chunk bases), and totals[e].  Called by all threads of a block with nw
// warps (nw <= 32); warp w owns a contiguous range of chunks.  part: shared [32][33].
__device__ __forceinline__ void scan_group(int32_t* cnt, int E, int C, int32_t* totals, int g,
                                           int nw, int w, int lane, int32_t (*part)[33]) {
  const int e = g * 32 + lane;
  const int per = (C + nw - 1) / nw;
  const int c0 = w * per, c1 = min(C, c0 + per);
  int sum = 0;
  if (e < E)
    for (int c = c0; c < c1; ++c) sum += __ldcg(cnt + static_cast<size_t>(c) * E + e);
  part[w][lane] = sum;
  __syncthreads();
  if (w == 0) {
    int run = 0;
    for (int i = 0; i < nw; ++i) {
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
  __syncthreads();
}

// offsets[0..E] = exclusive scan of totals[0..E), by all threads of one block (blockDim a
// multiple of 32, any E).  wsum: shared [32].
__device__ __forceinline__ void offsets_from_totals(const int32_t* totals, int E, int32_t* offsets,
                                                    int32_t* wsum) {
  const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int per = (E + nt - 1) / nt;
  const int i0 = tid * per, i1 = min(E, i0 + per);
  int local = 0;
  for (int i = i0; i < i1; ++i) local += __ldcg(totals + i);
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) wsum[w] = incl;
  __syncthreads();
  if (w == 0) {
    int v = lane < (nt >> 5) ? wsum[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += o;
    }
    wsum[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  int run = (w == 0 ? 0 : wsum[w - 1]) + incl - local;
  for (int i = i0; i < i1; ++i) {
    offsets[i] = run;
    run += __ldcg(totals + i);
  }
  if (tid == nt - 1) offsets[E] = wsum[(nt >> 5) - 1];
  __syncthreads();
}

// Slots and permutation of one 32-token chunk (one warp).  mask: E words of shared memory;
// bases: chunk bases from scan_group; offsets: expert offsets (global or shared).
__device__ __forceinline__ void assign_slots_chunk(uint32_t* mask,
                                                   const int32_t* __restrict__ topk_idx, int T,
                                                   int E, int k, int chunk,
                                                   const int32_t* __restrict__ bases,
                                                   const int32_t* offsets,
                                                   int32_t* __restrict__ perm_src,
                                                   int32_t* __restrict__ slot_of, int lane) {
  build_chunk_mask(mask, topk_idx, T, E, k, chunk, lane);
  const int t = chunk * kChunkTokens + lane;
  if (t < T) {
    const uint32_t below = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = __ldcg(topk_idx + static_cast<size_t>(t) * k + j);
      const int slot = offsets[e] + __ldcg(bases + static_cast<size_t>(chunk) * E + e) +
                       __popc(mask[e] & below);
      const int src = t * k + j;
      slot_of[src] = slot;
      perm_src[slot] = src;
    }
  }
  __syncwarp();
}

// Row copies of token t (one warp): its row of x (and of x_scales) goes to its k slots.
// Each 16-byte piece is read once; a lane keeps up to kV pieces in flight.
__device__ __forceinline__ void copy_token_rows(const uint8_t* __restrict__ x,
                                                const float* __restrict__ x_scales,
                                                int row_bytes, int nscale,
                                                const int32_t* __restrict__ slot_of, int t, int k,
                                                uint8_t* __restrict__ x_perm,
                                                float* __restrict__ x_perm_scales, int lane) {
  constexpr int kV = 8;
  int my_slot = 0;
  if (lane < k) my_slot = __ldcg(slot_of + static_cast<size_t>(t) * k + lane);
  int slots[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) slots[j] = __shfl_sync(0xffffffffu, my_slot, j);
  const int nvec = row_bytes / 16;
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * row_bytes);
  for (int v0 = lane; v0 < nvec; v0 += 32 * kV) {
    uint4 d[kV];
#pragma unroll
    for (int u = 0; u < kV; ++u)
      if (v0 + 32 * u < nvec) d[u] = __ldg(src + v0 + 32 * u);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j >= k) break;
      uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(slots[j]) * row_bytes);
#pragma unroll
      for (int u = 0; u < kV; ++u)
        if (v0 + 32 * u < nvec) dst[v0 + 32 * u] = d[u];
    }
  }
  if (x_scales != nullptr) {
    for (int v = lane; v < nscale; v += 32) {
      const float sv = __ldg(x_scales + static_cast<size_t>(t) * nscale + v);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j >= k) break;
        x_perm_scales[static_cast<size_t>(slots[j]) * nscale + v] = sv;
      }
    }
  }
}

// Token t's BF16 row, quantised to E4M3 on the way into its k slots: the activation
// quantisation that precedes dispatch, fused into the row copy (youleyou, "DeepSeek 模型更新
// 解读 Tile Kernels 与 DeepEP V2 新特性", Tile Kernels feature list, quantisation item: FP8
// per-block quantisation; jiqizhixin, "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了",
// FP8 x FP4 paragraph: FP8 activations).  Each 1x128 block gets the scale 2^n with n the
// smallest integer such that amax <= 448 * 2^n (n >= -126; an all-zero block gets 2^0 as
// the exponent rule gives), codes round to nearest even and saturate: the rule of the h
// requantisation.  BF16 values are exact in fp32 and the scaling by 2^-n is exact, so the
// codes depend on the input bits alone.  One warp per token (all 32 lanes call it); lane l
// holds elements 4l..4l+3 of a block, so loads read 256 contiguous bytes and each slot's
// codes are written as 128 contiguous bytes per block.
__device__ __forceinline__ void quant_copy_token_rows(const __nv_bfloat16* __restrict__ x, int H,
                                                      const int32_t* __restrict__ slot_of, int t,
                                                      int k, uint8_t* __restrict__ x_perm,
                                                      float* __restrict__ x_perm_scales,
                                                      int lane) {
  constexpr int kB = 4;  // blocks with loads in flight per lane
  int my_slot = 0;
  if (lane < k) my_slot = __ldcg(slot_of + static_cast<size_t>(t) * k + lane);
  int slots[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) slots[j] = __shfl_sync(0xffffffffu, my_slot, j);
  const int nb = H / 128;
  const uint2* src = reinterpret_cast<const uint2*>(x + static_cast<size_t>(t) * H);
  for (int b0 = 0; b0 < nb; b0 += kB) {
    uint2 raw[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u)
      raw[u] = b0 + u < nb ? __ldg(src + static_cast<size_t>(b0 + u) * 32 + lane) : make_uint2(0, 0);
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      if (b0 + u >= nb) break;  // warp-uniform
      const float2 f01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[u].x));
      const float2 f23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[u].y));
      const float a = fmaxf(fmaxf(fabsf(f01.x), fabsf(f01.y)), fmaxf(fabsf(f23.x), fabsf(f23.y)));
      // non-negative floats order like their bit patterns
      const float amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
      const int e = max(e4m3_scale_exponent(amax), -126);
      const float inv = exp2i(-e);
      const __nv_fp8x2_storage_t lo =
          __nv_cvt_float2_to_fp8x2(make_float2(f01.x * inv, f01.y * inv), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi =
          __nv_cvt_float2_to_fp8x2(make_float2(f23.x * inv, f23.y * inv), __NV_SATFINITE, __NV_E4M3);
      const uint32_t codes = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j >= k) break;  // warp-uniform
        reinterpret_cast<uint32_t*>(x_perm + static_cast<size_t>(slots[j]) * H +
                                    static_cast<size_t>(b0 + u) * 128)[lane] = codes;
      }
      if (lane < k) x_perm_scales[static_cast<size_t>(my_slot) * nb + b0 + u] = exp2i(e);
    }
  }
}

}  // namespace moe
