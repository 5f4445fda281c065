// Combine: out[t] = sum_{j<k} w[t, j] * y[slot_of[t*k + j]].
//
// The last step of the pages' pipeline puts the expert outputs back together (jiqizhixin,
// "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了", section "Mega MoE 是什么？", pipeline
// paragraph; youleyou, "DeepSeek 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", Tile Kernels
// feature list, routing item: fused reduce).  One warp per token gathers its k rows and sums
// them in rank order j in fp32, so the result is deterministic and needs no atomics.
// Shared by the combine kernel and the persistent forward kernel.
// HBM-bound: reads k rows of y per token, writes one output row, 16-byte accesses.
#pragma once

#include "common.cuh"

namespace moe {

__device__ __forceinline__ void load8(const void* base, size_t elem, int f32, float (&v)[8]) {
  if (f32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
    const float4 a = __ldcg(p), b = __ldcg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 u = __ldcg(reinterpret_cast<const uint4*>(
        static_cast<const __nv_bfloat16*>(base) + elem));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
}

// One warp computes out[t, :] (all 32 lanes call it together).
__device__ __forceinline__ void combine_token(const void* __restrict__ y, int y_f32,
                                              const int32_t* __restrict__ slot_of,
                                              const float* __restrict__ topk_w, int t, int k,
                                              int H, void* __restrict__ out, int out_f32,
                                              int lane) {
  int my_slot = 0;
  float my_w = 0.0f;
  if (lane < k) {
    my_slot = __ldcg(slot_of + static_cast<size_t>(t) * k + lane);
    my_w = __ldcg(topk_w + static_cast<size_t>(t) * k + lane);
  }
  const int nvec = H / 8;  // 8 elements per lane per step
  // The trip count is the same for every lane (shuffles below need the full warp); lanes
  // past the row's end only skip their loads and stores.
  for (int v0 = 0; v0 < nvec; v0 += 32) {
    const int v = v0 + lane;
    const bool act = v < nvec;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int slot = __shfl_sync(0xffffffffu, my_slot, j);
      const float w = __shfl_sync(0xffffffffu, my_w, j);
      if (act) {
        float r[8];
        load8(y, static_cast<size_t>(slot) * H + static_cast<size_t>(v) * 8, y_f32, r);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(w, r[i], acc[i]);
      }
    }
    if (!act) continue;
    const size_t o = static_cast<size_t>(t) * H + static_cast<size_t>(v) * 8;
    if (out_f32) {
      float4* p = reinterpret_cast<float4*>(static_cast<float*>(out) + o);
      p[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      p[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      uint4 u;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + o) = u;
    }
  }
}

}  // namespace moe
