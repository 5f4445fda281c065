// Host-side launchers shared between the library's translation units.  Each returns the
// cudaError_t of its launch(es); argument checking happens in api.cu before any of these
// is called.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

void count_launch(int n = 1);

// Dispatch workspace layout: per-chunk counts / bases [C][E] int32 and expert totals [E].
constexpr int kChunkTokens = 32;
inline size_t dispatch_ws_bytes(int T, int E) {
  size_t C = (static_cast<size_t>(T) + kChunkTokens - 1) / kChunkTokens;
  return ((C * E * 4 + 255) / 256) * 256 + ((static_cast<size_t>(E) * 4 + 255) / 256) * 256;
}

cudaError_t launch_route(const float* logits, const float* bias, int T, int E, int k, int score,
                         int renorm, int32_t* topk_idx, float* topk_w, cudaStream_t s,
                         int n_group = 1, int topk_group = 1, float scale = 1.0f);

cudaError_t launch_dispatch(const void* x, const float* x_scales, int row_bytes, int T, int H,
                            int E, int k, const int32_t* topk_idx, void* x_perm,
                            float* x_perm_scales, int32_t* offsets, int32_t* perm_src,
                            int32_t* slot_of, void* ws, cudaStream_t s,
                            bool quantize = false);

cudaError_t launch_combine(const void* y, int y_f32, const int32_t* slot_of, const float* topk_w,
                           int T, int k, int H, void* out, int out_f32, cudaStream_t s);

// Backward (BF16 layer) steps other than the expert GEMMs (backward.cu).
cudaError_t launch_transpose(const void* src, int elem_bytes, int E, int R, int C, void* dst,
                             cudaStream_t s);
cudaError_t launch_combine_backward(const void* dout, const void* y, const int32_t* slot_of,
                                    const float* topk_w, int T, int k, int H, void* dy_w,
                                    float* dgates, cudaStream_t s);
cudaError_t launch_gate_backward(const float* logits, const int32_t* topk_idx,
                                 const float* dgates, int T, int E, int k, int sigmoid,
                                 int renorm, float scale, float* dlogits, cudaStream_t s);
// Weight gradients on tensor cores (wgrad_tc.cu): pk = expert-padded segment starts, the
// slot-major operands transposed into [C, wgrad_pad_cols(S, E)] copies, then the GEMM.
size_t wgrad_pad_cols(int S, int E);
cudaError_t launch_wgrad_pad_offsets(const int32_t* offsets, int E, int32_t* pk, cudaStream_t s);
cudaError_t launch_pad_transpose(const void* X, int S, int C, const int32_t* offsets,
                                 const int32_t* pk, int E, void* Xt, cudaStream_t s);
cudaError_t launch_wgrad_tc(const void* At, const void* Bt, const int32_t* offsets,
                            const int32_t* pk, int S, int E, int M, int N, float* out, int* err,
                            cudaStream_t s);
cudaError_t launch_fill(float* p, size_t n, float v, cudaStream_t s);

struct FfnArgs {
  int act, wt;                 // moe_dtype
  const void* a;               // x_perm (linear-1) or h (linear-2)
  const float* a_scales;       // fp32 [S, K/128] or null
  const int32_t* offsets;      // [E+1]
  int S, H, I, E;
  const void* w;               // W1 or W2
  const void* w_scales;
  void* out;                   // h (linear-1) or y (linear-2)
  float* out_scales;           // h_scales (linear-1, E4M3) or null
  int* err;                    // device error word
  int scale_fmt = MOE_SCALE_POW2;  // moe_scale_fmt of the fp32 block scales
  const void* dh = nullptr;    // launch_linear1_dgate_tc: the gradient of h, BF16 [S, I]
};

cudaError_t launch_linear1_simt(const FfnArgs& a, cudaStream_t s);
cudaError_t launch_linear2_simt(const FfnArgs& a, cudaStream_t s);

// tcgen05 path; returns cudaErrorNotSupported for dtype pairs it does not cover.
cudaError_t launch_linear1_tc(const FfnArgs& a, cudaStream_t s);
// The backward form of linear-1 (BF16): recomputes the pre-activations g, u = x . W1^T of
// each slot on the tensor cores and writes out = dG [S, 2I] (dg in columns [0, I), du in
// [I, 2I)) from them and a.dh, the gradient of h = silu(g) u, without storing g or u.
cudaError_t launch_linear1_dgate_tc(const FfnArgs& a, cudaStream_t s);
cudaError_t launch_linear2_tc(const FfnArgs& a, cudaStream_t s);

// 2-D K-major tensor map: rows x K, box {128-byte K slice, 128 rows}, 128-byte swizzle.
// fmt: 0 = BF16, 1 = 8-bit, 2 = E2M1 (expanded to one byte per element in shared memory).
bool make_kmajor_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K, int fmt,
                     uint32_t box_rows = 128);

// The whole layer in one persistent cooperative launch (tensor-core formats only);
// returns cudaErrorNotSupported when the layer cannot run that way.
struct ForwardArgs {
  const void* x;
  const float* x_scales;
  const float* logits;
  const float* bias;
  int sigmoid, renorm, T, H, E, k, I;
  int n_group = 1, topk_group = 1;  // group-limited routing (1, 1: plain)
  float scale = 1.0f;               // routed scaling factor
  int act, wt;
  const void* w1;
  const void* w1_scales;
  const void* w2;
  const void* w2_scales;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* offsets;
  int32_t* perm_src;
  int32_t* slot_of;
  void* x_perm;
  float* x_perm_scales;
  int32_t* cnt;      // dispatch chunk counts [C][E]
  int32_t* totals;   // [E]
  void* h;
  float* h_scales;
  void* y;
  void* out;
  uint32_t* bar;     // grid barrier words (zeroed by the launcher)
  int* err;
};
cudaError_t launch_forward_fused(const ForwardArgs& a, cudaStream_t s);

// Self-test kernels whose bounded waits run out by construction (selftest.cu).
cudaError_t launch_wait_selftest(int kind, int* err, cudaStream_t s);

int* device_error_word();   // device address of the calling device's error word
int gemm_tile_mode();
// Tile shape for a grouped GEMM over S rows and E experts: 1 single, 2 pair, 3 small (32-row
// m-blocks).  allow_pair = false where only single-CTA shapes exist (the persistent kernel).
int gemm_tile_shape(int act, int S, int E, bool allow_pair);       // 0 automatic, 1 single-CTA tiles, 2 CTA-pair tiles
int num_sms();

// Shape checks shared by the dispatch entry points (and the layer-level calls): T, H, E, k
// within the supported ranges.  Returns MOE_OK, MOE_ERR_INVALID_ARG or MOE_ERR_UNSUPPORTED.
moe_status check_dispatch_shapes(int T, int H, int E, int k);

}  // namespace moe
