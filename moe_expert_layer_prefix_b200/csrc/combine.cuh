// Combine: out[t] = sum_{j<k} w[t, j] * y[slot_of[t*k + j]].
//
// The last step of the pages' pipeline puts the expert outputs back together (jiqizhixin,
// "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了", section "Mega MoE 是什么？", pipeline
// paragraph; youleyou, "DeepSeek 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", Tile Kernels
// feature list, routing item: fused reduce).  A warp takes a chunk of one token's columns,
// gathers them from the token's k rows and sums in rank order j in fp32, so the result is
// deterministic and needs no atomics.
// Shared by the combine kernel and the persistent forward kernel.
// HBM-bound: reads k rows of y per token, writes one output row, 16-byte accesses.
#pragma once

#include "common.cuh"

namespace moe {

// Columns of a token are handed out in chunks of 32 * kV vectors of 8 columns (one warp
// iteration), so that few tokens still spread over many warps.
template <int kV>
__host__ __device__ constexpr int combine_chunks(int H) {
  return (H / 8 + 32 * kV - 1) / (32 * kV);
}

// One warp computes out[t, 8*v_begin : 8*v_end] (all 32 lanes call it together; v_begin is a
// multiple of 32 * kV).  y and out are BF16, or fp32 for the fp32 layer.  Each lane owns 8
// consecutive columns per pass and a warp iteration covers kV passes; the k source rows are
// read as groups of kJ x kV independent 16-byte loads issued back to back (raw words,
// converted only afterwards), so a warp keeps many loads in flight even when only a few
// warps per SM run it.
template <bool kF32, int kV = 1>
__device__ __forceinline__ void combine_token(const void* __restrict__ y,
                                              const int32_t* __restrict__ slot_of,
                                              const float* __restrict__ topk_w, int t, int k,
                                              int H, void* __restrict__ out, int lane,
                                              int v_begin, int v_end) {
  constexpr int kJ = 8;
  constexpr int kWords = kF32 ? 2 : 1;  // 16-byte words per 8 columns
  int my_slot = 0;
  float my_w = 0.0f;
  if (lane < k) {
    my_slot = __ldcg(slot_of + static_cast<size_t>(t) * k + lane);
    my_w = __ldcg(topk_w + static_cast<size_t>(t) * k + lane);
  }
  const int nvec = v_end < H / 8 ? v_end : H / 8;
  const uint4* y4 = static_cast<const uint4*>(y);
  const size_t row_words = static_cast<size_t>(H) / 8 * kWords;
  // The trip counts are the same for every lane (the shuffles need the full warp); lanes
  // past the row's end read column 0 and drop the result.
  for (int v0 = v_begin; v0 < nvec; v0 += 32 * kV) {
    size_t col[kV];
#pragma unroll
    for (int p = 0; p < kV; ++p) {
      const int v = v0 + 32 * p + lane;
      col[p] = static_cast<size_t>(v < nvec ? v : 0) * kWords;
    }
    float acc[kV][8];
#pragma unroll
    for (int p = 0; p < kV; ++p)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[p][i] = 0.0f;
    for (int j0 = 0; j0 < k; j0 += kJ) {
      uint4 raw[kJ][kV][kWords];
      float w[kJ];
      int slot[kJ];
#pragma unroll
      for (int jj = 0; jj < kJ; ++jj) {
        slot[jj] = __shfl_sync(0xffffffffu, my_slot, (j0 + jj) & 31);
        w[jj] = __shfl_sync(0xffffffffu, my_w, (j0 + jj) & 31);
      }
#pragma unroll
      for (int jj = 0; jj < kJ; ++jj) {
        // rows past the token's k are not loaded at all (k = 2 would otherwise re-read a
        // row six times per pass)
        if (j0 + jj >= k) break;  // warp-uniform
        const uint4* row = y4 + static_cast<size_t>(slot[jj]) * row_words;
#pragma unroll
        for (int p = 0; p < kV; ++p)
#pragma unroll
          for (int q = 0; q < kWords; ++q) raw[jj][p][q] = __ldcg(row + col[p] + q);
      }
#pragma unroll
      for (int jj = 0; jj < kJ; ++jj) {
        if (j0 + jj >= k) break;  // warp-uniform
#pragma unroll
        for (int p = 0; p < kV; ++p) {
          float r[8];
          if constexpr (kF32) {
            const float* f = reinterpret_cast<const float*>(raw[jj][p]);
#pragma unroll
            for (int i = 0; i < 8; ++i) r[i] = f[i];
          } else {
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[jj][p][0]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = __bfloat1622float2(h2[i]);
              r[2 * i] = f.x;
              r[2 * i + 1] = f.y;
            }
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[p][i] = fmaf(w[jj], r[i], acc[p][i]);
        }
      }
    }
#pragma unroll
    for (int p = 0; p < kV; ++p) {
      const int v = v0 + 32 * p + lane;
      if (v >= nvec) continue;
      const size_t o = static_cast<size_t>(t) * H + static_cast<size_t>(v) * 8;
      if constexpr (kF32) {
        float4* q = reinterpret_cast<float4*>(static_cast<float*>(out) + o);
        q[0] = make_float4(acc[p][0], acc[p][1], acc[p][2], acc[p][3]);
        q[1] = make_float4(acc[p][4], acc[p][5], acc[p][6], acc[p][7]);
      } else {
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[p][2 * i], acc[p][2 * i + 1]);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + o) = u;
      }
    }
  }
}

}  // namespace moe
