// Expert FFN on CUDA cores, one block per dispatch slot.
//
// This is the path for the fp32 layer, whose precision the tensor-core kinds used
// elsewhere cannot hold (tf32 would round the inputs).  It handles every format, so it also
// serves as an independent second implementation of linear-1 / linear-2 in the tests.
//   linear-1: gate = x . W1[e, i], up = x . W1[e, I+i], h_i = silu(gate) * up, h stored in
//             the activation format (E4M3: power-of-two scale per 1x128 block);
//   linear-2: y_c = h . W2[e, c], stored BF16 (F32 for the fp32 layer).
// (jiqizhixin, "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了", section "Mega MoE 是什么？",
//  pipeline paragraph and FP8 x FP4 paragraph.)
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  __nv_fp8_e4m3 v;
  v.__x = c;
  return static_cast<float>(v);
}

__device__ __forceinline__ float e2m1_to_f32(uint32_t code) {
  const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  const float m = mag[code & 7u];
  return (code & 8u) ? -m : m;
}

// Element (r, c) of one expert's weight matrix [R, C] in format wt, dequantised.
__device__ __forceinline__ float weight_at(const void* w, const void* ws, int wt, int R, int C,
                                           int r, int c) {
  switch (wt) {
    case MOE_F32:
      return static_cast<const float*>(w)[static_cast<size_t>(r) * C + c];
    case MOE_BF16:
      return __bfloat162float(static_cast<const __nv_bfloat16*>(w)[static_cast<size_t>(r) * C + c]);
    case MOE_E4M3: {
      const float s = static_cast<const float*>(ws)[static_cast<size_t>(r / 128) * (C / 128) + c / 128];
      return e4m3_to_f32(static_cast<const uint8_t*>(w)[static_cast<size_t>(r) * C + c]) * s;
    }
    default: {  // E2M1
      const uint8_t b = static_cast<const uint8_t*>(w)[static_cast<size_t>(r) * (C / 2) + c / 2];
      const uint8_t sb = static_cast<const uint8_t*>(ws)[static_cast<size_t>(r) * (C / 32) + c / 32];
      return e2m1_to_f32((c & 1) ? (b >> 4) : (b & 15)) * exp2i(static_cast<int>(sb) - 127);
    }
  }
}

__device__ __forceinline__ float act_at(const void* a, const float* sc, int act, int C,
                                        size_t row, int c) {
  switch (act) {
    case MOE_F32:
      return static_cast<const float*>(a)[row * C + c];
    case MOE_BF16:
      return __bfloat162float(static_cast<const __nv_bfloat16*>(a)[row * C + c]);
    default:
      return e4m3_to_f32(static_cast<const uint8_t*>(a)[row * C + c]) * sc[row * (C / 128) + c / 128];
  }
}

__device__ int expert_of_slot(const int32_t* offsets, int E, int p) {
  int lo = 0, hi = E;  // offsets[lo] <= p < offsets[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(offsets + mid) <= p) lo = mid; else hi = mid;
  }
  return lo;
}

// Stores a row of fp32 values `v` [n] in format act (+ one scale per 128 for E4M3).
// Called by the whole block; v in shared memory.
__device__ void store_row(const float* v, int n, int act, void* out, float* out_scales,
                          size_t row) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (act == MOE_F32) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) static_cast<float*>(out)[row * n + i] = v[i];
  } else if (act == MOE_BF16) {
    for (int i = threadIdx.x; i < n; i += blockDim.x)
      static_cast<__nv_bfloat16*>(out)[row * n + i] = __float2bfloat16_rn(v[i]);
  } else {
    for (int b = w; b < n / 128; b += nw) {
      float amax = 0.0f;
      for (int i = lane; i < 128; i += 32) amax = fmaxf(amax, fabsf(v[b * 128 + i]));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const int e = max(e4m3_scale_exponent(amax), -126);
      const float inv = exp2i(-e > 127 ? 127 : -e);
      for (int i = lane; i < 128; i += 32) {
        const __nv_fp8_e4m3 q(v[b * 128 + i] * inv);  // RNE, saturating to +-448
        static_cast<uint8_t*>(out)[row * n + b * 128 + i] = q.__x;
      }
      if (lane == 0) out_scales[row * (n / 128) + b] = exp2i(e);
    }
  }
}

__global__ void __launch_bounds__(256) linear1_simt_kernel(FfnArgs a) {
  extern __shared__ float sm[];
  float* xs = sm;              // [H]
  float* hs = sm + a.H;        // [I]
  const int p = blockIdx.x;
  const int e = expert_of_slot(a.offsets, a.E, p);
  for (int c = threadIdx.x; c < a.H; c += blockDim.x)
    xs[c] = act_at(a.a, a.a_scales, a.act, a.H, static_cast<size_t>(p), c);
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const size_t wsz = a.wt == MOE_E2M1 ? static_cast<size_t>(2 * a.I) * a.H / 2
                                      : static_cast<size_t>(2 * a.I) * a.H;
  const size_t esz = a.wt == MOE_F32 ? 4 : a.wt == MOE_BF16 ? 2 : 1;
  const char* we = static_cast<const char*>(a.w) + static_cast<size_t>(e) * wsz * esz;
  const char* wse = nullptr;
  if (a.wt == MOE_E4M3)
    wse = static_cast<const char*>(a.w_scales) + static_cast<size_t>(e) * (2 * a.I / 128) * (a.H / 128) * 4;
  if (a.wt == MOE_E2M1)
    wse = static_cast<const char*>(a.w_scales) + static_cast<size_t>(e) * (2 * a.I) * (a.H / 32);
  for (int i = w; i < a.I; i += nw) {
    float g = 0.0f, u = 0.0f;
    for (int c = lane; c < a.H; c += 32) {
      g = fmaf(xs[c], weight_at(we, wse, a.wt, 2 * a.I, a.H, i, c), g);
      u = fmaf(xs[c], weight_at(we, wse, a.wt, 2 * a.I, a.H, a.I + i, c), u);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, off);
      u += __shfl_xor_sync(0xffffffffu, u, off);
    }
    if (lane == 0) hs[i] = g / (1.0f + expf(-g)) * u;
  }
  __syncthreads();
  store_row(hs, a.I, a.act, a.out, a.out_scales, static_cast<size_t>(p));
}

__global__ void __launch_bounds__(256) linear2_simt_kernel(FfnArgs a) {
  extern __shared__ float sm[];
  float* hs = sm;  // [I]
  const int p = blockIdx.x;
  const int e = expert_of_slot(a.offsets, a.E, p);
  for (int c = threadIdx.x; c < a.I; c += blockDim.x)
    hs[c] = act_at(a.a, a.a_scales, a.act, a.I, static_cast<size_t>(p), c);
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const size_t wsz = a.wt == MOE_E2M1 ? static_cast<size_t>(a.H) * a.I / 2
                                      : static_cast<size_t>(a.H) * a.I;
  const size_t esz = a.wt == MOE_F32 ? 4 : a.wt == MOE_BF16 ? 2 : 1;
  const char* we = static_cast<const char*>(a.w) + static_cast<size_t>(e) * wsz * esz;
  const char* wse = nullptr;
  if (a.wt == MOE_E4M3)
    wse = static_cast<const char*>(a.w_scales) + static_cast<size_t>(e) * (a.H / 128) * (a.I / 128) * 4;
  if (a.wt == MOE_E2M1)
    wse = static_cast<const char*>(a.w_scales) + static_cast<size_t>(e) * a.H * (a.I / 32);
  const bool f32 = a.act == MOE_F32;
  for (int c = w; c < a.H; c += nw) {
    float acc = 0.0f;
    for (int i = lane; i < a.I; i += 32) acc = fmaf(hs[i], weight_at(we, wse, a.wt, a.H, a.I, c, i), acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      const size_t o = static_cast<size_t>(p) * a.H + c;
      if (f32) static_cast<float*>(a.out)[o] = acc;
      else static_cast<__nv_bfloat16*>(a.out)[o] = __float2bfloat16_rn(acc);
    }
  }
}

}  // namespace

cudaError_t launch_linear1_simt(const FfnArgs& a, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(a.H + a.I) * 4;
  cudaError_t err = cudaFuncSetAttribute(linear1_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  count_launch();
  linear1_simt_kernel<<<a.S, 256, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_linear2_simt(const FfnArgs& a, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(a.I) * 4;
  cudaError_t err = cudaFuncSetAttribute(linear2_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  count_launch();
  linear2_simt_kernel<<<a.S, 256, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
