// Backward of the expert layer (BF16 layer): the steps that are not expert GEMMs.
//
// The pages mention training only in passing: youleyou, "DeepSeek 模型更新解读 Tile Kernels 与
// DeepEP V2 新特性", section "Tile Kernels：逼近硬件极限的底层优化", feature list, the
// batched-transpose item and the model-layer item (wrappers that make the kernels trainable
// layers).  The gradients are those of the layer's definition with the top-k selection held
// fixed (it is piecewise constant in the logits):
//   combine:  dy_w[slot(t, j)] = w[t, j] * dout[t],   dgate[t, j] = dout[t] . y[slot(t, j)]
//   router:   d logits from dgate through the gate function (softmax over the selected
//             logits, the full softmax without renormalisation, the renormalised sigmoid)
//   SwiGLU:   dg = dh * u * s * (1 + g * (1 - s)),  du = dh * g * s,  s = sigmoid(g)
//   weights:  dW1_e = dG_e^T x_e,  dW2_e = dy_w,e^T h_e  (sums over the expert's slots)
// The activation gradients (dh = dy_w W2, dx_slot = dG W1) and the recomputed
// pre-activations (G = x W1^T) run on the forward pass's tensor-core expert GEMM, given the
// weights in the layout it reads (transpose_kernel below makes the transposed copies); the
// weight gradients run on tensor cores in wgrad_tc.cu.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// dst[e] = src[e]^T for src [E, R, C] (row-major): 32 x 32 tiles through shared memory, so
// that both the reads and the writes run along rows.
template <typename T>
__global__ void __launch_bounds__(256) transpose_kernel(const T* __restrict__ src, int R, int C,
                                                        T* __restrict__ dst) {
  __shared__ T tile[32][33];
  const size_t base = static_cast<size_t>(blockIdx.z) * R * C;
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int r = r0 + ty + i, c = c0 + tx;
    if (r < R && c < C) tile[ty + i][tx] = src[base + static_cast<size_t>(r) * C + c];
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int c = c0 + ty + i, r = r0 + tx;
    if (r < R && c < C) dst[base + static_cast<size_t>(c) * R + r] = tile[tx][ty + i];
  }
}

// One warp per token: for each of its k slots, dgate = dout[t] . y[slot] (fp32, lanes in a
// fixed order, then a butterfly: deterministic) and dy_w[slot] = BF16(w * dout[t]).
__global__ void __launch_bounds__(256) combine_backward_kernel(
    const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ y,
    const int32_t* __restrict__ slot_of, const float* __restrict__ topk_w, int T, int k, int H,
    __nv_bfloat16* __restrict__ dy_w, float* __restrict__ dgates) {
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int nvec = H / 8;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nw) {
    const uint4* drow = reinterpret_cast<const uint4*>(dout + static_cast<size_t>(t) * H);
    for (int j = 0; j < k; ++j) {
      const int slot = __ldg(slot_of + static_cast<size_t>(t) * k + j);
      const float w = __ldg(topk_w + static_cast<size_t>(t) * k + j);
      const uint4* yrow = reinterpret_cast<const uint4*>(y + static_cast<size_t>(slot) * H);
      uint4* orow = reinterpret_cast<uint4*>(dy_w + static_cast<size_t>(slot) * H);
      float acc = 0.0f;
      for (int v = lane; v < nvec; v += 32) {
        const uint4 d = __ldg(drow + v), yy = __ldg(yrow + v);
        const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&d);
        const __nv_bfloat162* y2 = reinterpret_cast<const __nv_bfloat162*>(&yy);
        uint4 o;
        __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 df = __bfloat1622float2(d2[i]);
          const float2 yf = __bfloat1622float2(y2[i]);
          acc = fmaf(df.x, yf.x, acc);
          acc = fmaf(df.y, yf.y, acc);
          o2[i] = __floats2bfloat162_rn(w * df.x, w * df.y);
        }
        orow[v] = o;
      }
      acc = warp_sum(acc);
      if (lane == 0) dgates[static_cast<size_t>(t) * k + j] = acc;
    }
  }
}

// One warp per token: d logits [E] from the k gate gradients (lane j holds slot j).
__global__ void __launch_bounds__(256) gate_backward_kernel(
    const float* __restrict__ logits, const int32_t* __restrict__ topk_idx,
    const float* __restrict__ dgates, int T, int E, int k, int sigmoid, int renorm, float scale,
    float* __restrict__ dlogits) {
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nw) {
    const float* l = logits + static_cast<size_t>(t) * E;
    float* out = dlogits + static_cast<size_t>(t) * E;
    const bool sel = lane < k;
    const int ej = sel ? __ldg(topk_idx + static_cast<size_t>(t) * k + lane) : 0;
    const float lj = sel ? __ldg(l + ej) : -INFINITY;
    const float dw = sel ? __ldg(dgates + static_cast<size_t>(t) * k + lane) : 0.0f;
    float g = 0.0f;
    if (!sigmoid && !renorm) {
      // w_j = scale * p_{e_j} with p the softmax over all E logits:
      // dl_m = scale * p_m * ([m selected] dw_m - sum_j p_{e_j} dw_j)
      float m = -INFINITY;
      for (int e = lane; e < E; e += 32) m = fmaxf(m, __ldg(l + e));
      m = warp_max(m);
      float z = 0.0f;
      for (int e = lane; e < E; e += 32) z += expf(__ldg(l + e) - m);
      const float Z = warp_sum(z);
      const float pj = sel ? expf(lj - m) / Z : 0.0f;
      const float sd = warp_sum(pj * dw);
      for (int e = lane; e < E; e += 32) out[e] = -scale * (expf(__ldg(l + e) - m) / Z) * sd;
      g = scale * pj * (dw - sd);
    } else {
      if (!sigmoid) {
        // w = scale * softmax over the selected logits: dl_j = scale * p_j (dw_j - sum p dw)
        const float m = warp_max(lj);
        const float z = sel ? expf(lj - m) : 0.0f;
        const float p = z / warp_sum(z);
        g = scale * p * (dw - warp_sum(p * dw));
      } else {
        // s = sigmoid(l); w = scale * s (no renorm) or scale * s / sum_sel s
        const float s = sel ? 1.0f / (1.0f + expf(-lj)) : 0.0f;
        float ds = dw;
        if (renorm) {
          const float tot = warp_sum(s);
          const float q = s / tot;
          ds = (dw - warp_sum(q * dw)) / tot;
        }
        g = scale * ds * s * (1.0f - s);
      }
      for (int e = lane; e < E; e += 32) out[e] = 0.0f;
    }
    __syncwarp();  // the row's plain values are in place before the selected ones
    if (sel) out[ej] = g;
    __syncwarp();
  }
}

// dG = [dg | du] from the recomputed pre-activations G = [g | u] [S, 2I] and dh [S, I], in
// fp32, stored BF16; 8 columns per thread.
__global__ void fill_kernel(float* __restrict__ p, size_t n, float v) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[i] = v;
}

inline unsigned warp_grid(long warps_needed) {
  const long blocks = (warps_needed + 7) / 8;
  const long cap = static_cast<long>(num_sms()) * 16;
  return static_cast<unsigned>(blocks < 1 ? 1 : (blocks < cap ? blocks : cap));
}

}  // namespace

cudaError_t launch_transpose(const void* src, int elem_bytes, int E, int R, int C, void* dst,
                             cudaStream_t s) {
  const dim3 grid((C + 31) / 32, (R + 31) / 32, E), block(256);
  count_launch();
  switch (elem_bytes) {
    case 1:
      transpose_kernel<uint8_t><<<grid, block, 0, s>>>(static_cast<const uint8_t*>(src), R, C,
                                                       static_cast<uint8_t*>(dst));
      break;
    case 2:
      transpose_kernel<uint16_t><<<grid, block, 0, s>>>(static_cast<const uint16_t*>(src), R, C,
                                                        static_cast<uint16_t*>(dst));
      break;
    default:
      transpose_kernel<uint32_t><<<grid, block, 0, s>>>(static_cast<const uint32_t*>(src), R, C,
                                                        static_cast<uint32_t*>(dst));
  }
  return cudaGetLastError();
}

cudaError_t launch_combine_backward(const void* dout, const void* y, const int32_t* slot_of,
                                    const float* topk_w, int T, int k, int H, void* dy_w,
                                    float* dgates, cudaStream_t s) {
  count_launch();
  combine_backward_kernel<<<warp_grid(T), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(y), slot_of,
      topk_w, T, k, H, static_cast<__nv_bfloat16*>(dy_w), dgates);
  return cudaGetLastError();
}

cudaError_t launch_gate_backward(const float* logits, const int32_t* topk_idx,
                                 const float* dgates, int T, int E, int k, int sigmoid,
                                 int renorm, float scale, float* dlogits, cudaStream_t s) {
  count_launch();
  gate_backward_kernel<<<warp_grid(T), 256, 0, s>>>(logits, topk_idx, dgates, T, E, k, sigmoid,
                                                    renorm, scale, dlogits);
  return cudaGetLastError();
}

cudaError_t launch_fill(float* p, size_t n, float v, cudaStream_t s) {
  const size_t blocks = (n + 255) / 256;
  const size_t cap = static_cast<size_t>(num_sms()) * 8;
  count_launch();
  fill_kernel<<<static_cast<unsigned>(blocks < 1 ? 1 : (blocks < cap ? blocks : cap)), 256, 0,
                s>>>(p, n, v);
  return cudaGetLastError();
}

}  // namespace moe
