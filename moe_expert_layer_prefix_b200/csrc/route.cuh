// Router, per token: one warp selects the k best experts and writes their gates (shared by
// the router kernel and the persistent forward kernel).
//
// Gating as the source pages list it (youleyou, "DeepSeek 模型更新解读 Tile Kernels 与 DeepEP
// V2 新特性", section "Tile Kernels：逼近硬件极限的底层优化": gating = top-k expert
// selection with scoring; routing = weight normalisation).  The scoring rules are the
// library's reading of that item:
//   softmax: key = logit; gate_j = exp(l_j - l_0) / sum over the selected (renorm) or over
//            all experts (no renorm), l_0 the largest logit;
//   sigmoid: s = 1 / (1 + exp(-l)) evaluated as a fixed sequence of correctly rounded fp32
//            operations (the exponential below), key = s + bias_e;
//            gate_j = s_j / sum of selected s (renorm) or s_j.
// Rank order: key descending, equal keys -> lower expert id.
//
// HBM-bound: each token's E logits are read once, coalesced across the warp.
#pragma once

#include "common.cuh"

namespace moe {

// fp32 exponential by Cody-Waite range reduction (two-part ln 2) and the degree-7 Taylor
// polynomial of the reduced argument, every step a separately rounded fp32 operation
// (Cody & Waite, "Software Manual for the Elementary Functions", 1980).  Used only to form
// the sigmoid router's selection keys, so that the selection is a function of the fp32
// keys alone.
__device__ __forceinline__ float exp_keys_f32(float x) {
  const float kLog2e = 1.44269504088896340736f;
  const float kLn2Hi = 0.693145751953125f;
  const float kLn2Lo = 1.42860682030941723212e-6f;
  x = fminf(fmaxf(x, -80.0f), 80.0f);
  const float n = rintf(__fmul_rn(x, kLog2e));
  float r = __fsub_rn(x, __fmul_rn(n, kLn2Hi));
  r = __fsub_rn(r, __fmul_rn(n, kLn2Lo));
  float p = 1.98412698412698412698e-4f;                 // 1/7!
  p = __fadd_rn(__fmul_rn(p, r), 1.38888888888888888889e-3f);  // 1/6!
  p = __fadd_rn(__fmul_rn(p, r), 8.33333333333333333333e-3f);  // 1/5!
  p = __fadd_rn(__fmul_rn(p, r), 4.16666666666666666667e-2f);  // 1/4!
  p = __fadd_rn(__fmul_rn(p, r), 1.66666666666666666667e-1f);  // 1/3!
  p = __fadd_rn(__fmul_rn(p, r), 0.5f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  return __fmul_rn(p, exp2i(static_cast<int>(n)));
}

__device__ __forceinline__ float sigmoid_keys_f32(float l) {
  return __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_keys_f32(-l)));
}

// Order-preserving integer of an fp32 selection key (-0 taken as +0, so that equal keys give
// equal words; NaNs order by their bit patterns).
__device__ __forceinline__ uint32_t ord_key(float key) {
  const uint32_t u = __float_as_uint(__fadd_rn(key, 0.0f));
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// A candidate as one 64-bit word ordered like (key, id): the ordered key in the high half, the
// complemented id in the low half (lower id wins a tie).  0 is below every candidate.
__device__ __forceinline__ uint64_t pack_cand(uint32_t ku, int e) {
  return (static_cast<uint64_t>(ku) << 32) | static_cast<uint32_t>(~e);
}

// Per-warp shared-memory scratch of route_token: kRouteCand packed candidates, then the k
// selected ids.
constexpr int kRouteCand = 128;
constexpr int kRouteScratchBytes = kRouteCand * 8 + 32 * 4;

// One warp selects the k experts of token t and writes topk_idx[t, :], topk_w[t, :].
// Lanes hold experts lane, lane+32, ...; all 32 lanes must call it together, each warp with
// its own kRouteScratchBytes of 8-byte aligned shared memory.
// Group-limited selection (n_group > 1, groups of G = E / n_group experts with G a multiple
// of 32): a group's score is the fp32 sum of its two largest keys, the topk_group best groups
// (equal scores -> lower group) are kept and the k experts are chosen among theirs only.
// Gates are multiplied by `scale` (the routed scaling factor).  n_group = 1, scale = 1 is
// the plain router.
// Token t's logits, lane l holding experts l, l + 32, ... (0 past E).
template <int NPL>
__device__ __forceinline__ void route_load(const float* __restrict__ logits, int t, int E,
                                           int lane, float (&l)[NPL]) {
  const float* row = logits + static_cast<size_t>(t) * E;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    l[i] = e < E ? __ldg(row + e) : 0.0f;
  }
}

template <int NPL>  // experts per lane (E <= 32 * NPL)
__device__ __forceinline__ void route_select(const float (&lg)[NPL],
                                             const float* __restrict__ logits,
                                             const float* __restrict__ bias, int t, int E, int k,
                                             int sigmoid, int renorm,
                                             int32_t* __restrict__ topk_idx,
                                             float* __restrict__ topk_w, int lane,
                                             uint8_t* scratch, int n_group, int topk_group,
                                             float scale) {
  const float* row = logits + static_cast<size_t>(t) * E;

  float key[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const float l = lg[i];
      key[i] = sigmoid ? __fadd_rn(sigmoid_keys_f32(l), bias ? __ldg(bias + e) : 0.0f) : l;
    } else {
      key[i] = -INFINITY;
    }
  }

  // Groups.  Lane l holds experts l + 32i, so with G a multiple of 32 a group is sg = G / 32
  // consecutive slots i of every lane: each lane keeps a running top-2 over the group's
  // slots and the warp merges them at the group's last slot; slots of groups that are not
  // kept are not candidates.
  uint32_t taken = 0;
  if (n_group > 1) {
    const int sg = E / n_group / 32;
    float gsc[NPL];    // at a group's last slot: the group's score
    float a1 = -INFINITY, a2 = -INFINITY;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      gsc[i] = -INFINITY;
      if (32 * i < E) {
        const float x = key[i];
        a2 = fmaxf(a2, fminf(a1, x));
        a1 = fmaxf(a1, x);
        if ((i + 1) % sg == 0) {  // warp-uniform
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            const float b1v = __shfl_xor_sync(0xffffffffu, a1, off);
            const float b2v = __shfl_xor_sync(0xffffffffu, a2, off);
            const float hi = fmaxf(a1, b1v);
            a2 = fmaxf(fminf(a1, b1v), fmaxf(a2, b2v));
            a1 = hi;
          }
          gsc[i] = __fadd_rn(a1, a2);
          a1 = a2 = -INFINITY;
        }
      }
    }
    uint32_t keep = 0;  // bit i: slot i is the last slot of a kept group
    for (int r = 0; r < topk_group; ++r) {
      float best = 0.0f;
      int bi = -1;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        if (32 * i < E && (i + 1) % sg == 0 && !((keep >> i) & 1u) &&
            (bi < 0 || gsc[i] > best)) {
          best = gsc[i];
          bi = i;
        }
      }
      if (bi >= 0) keep |= 1u << bi;
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int last = (i / sg) * sg + sg - 1;
      if (!((keep >> last) & 1u)) taken |= 1u << i;
    }
  }

  // Ordered keys of this lane's eligible experts (0 marks an ineligible slot; the ordered
  // key of an eligible one may be 0 too, which only ever adds candidates below).
  uint32_t elig = 0;
  uint32_t ku[NPL];
  uint32_t m = 0;  // this lane's largest ordered key
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const bool ok = lane + 32 * i < E && !((taken >> i) & 1u);
    ku[i] = ok ? ord_key(key[i]) : 0u;
    elig |= static_cast<uint32_t>(ok) << i;
    m = max(m, ku[i]);
  }

  // Selection.  A lower bound of the k-th best key: the k-th largest of the 32 lane maxima
  // (bitonic sort of the lane maxima across the warp).  When it is above 0, k lanes hold a
  // key at or above it, so every one of the k best is a key at or above it; at 0 every
  // eligible expert is a candidate.  The candidates (a few dozen on router logits) are
  // compacted into shared memory in (slot, lane) order and each is ranked by the number of
  // candidates above it in (key, id) order, which is exact and has no ties (ids differ).
  uint32_t v = m;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint32_t o = __shfl_xor_sync(0xffffffffu, v, stride);
      const bool lower = (lane & stride) == 0, up = (lane & size) == 0;
      v = (lower == up) ? min(v, o) : max(v, o);
    }
  }
  const uint32_t bound = __shfl_sync(0xffffffffu, v, 32 - k);  // ascending across lanes

  uint64_t* cand = reinterpret_cast<uint64_t*>(scratch);
  int32_t* sel = reinterpret_cast<int32_t*>(scratch + kRouteCand * 8);
  const uint32_t below = (1u << lane) - 1u;
  int n = 0;  // candidates so far (warp-uniform)
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const bool is_c = ((elig >> i) & 1u) && ku[i] >= bound;
    const uint32_t bal = __ballot_sync(0xffffffffu, is_c);
    if (is_c) {
      const int pos = n + __popc(bal & below);
      if (pos < kRouteCand) cand[pos] = pack_cand(ku[i], lane + 32 * i);
    }
    n += __popc(bal);
  }
  __syncwarp();

  int my_idx = 0;  // lane j keeps the j-th selection
  if (n <= kRouteCand) {
    for (int j = lane; j < n; j += 32) {
      const uint64_t cj = cand[j];
      int r = 0;
#pragma unroll 4
      for (int i = 0; i < n; ++i) r += cand[i] > cj;
      if (r < k) sel[r] = static_cast<int>(~static_cast<uint32_t>(cj));
    }
    __syncwarp();
    if (lane < k) my_idx = sel[lane];
  } else {
    // Many keys tie at the bound (constant logits, say): k rounds of a warp maximum over
    // each lane's best four untaken candidates; the winning lane moves its list up and
    // rescans its NPL experts only once all four are taken.
    constexpr int kC = 4;
    uint64_t c[kC];
    int n_c = 0;  // valid entries of c
    auto scan = [&]() {
#pragma unroll
      for (int q = 0; q < kC; ++q) c[q] = 0;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        if ((elig >> i) & 1u) {
          uint64_t y = pack_cand(ku[i], lane + 32 * i);
          if (y > c[kC - 1]) {  // insert, keeping c sorted
#pragma unroll
            for (int q = 0; q < kC; ++q) {
              if (y > c[q]) {
                const uint64_t t0 = c[q];
                c[q] = y;
                y = t0;
              }
            }
          }
        }
      }
      n_c = 0;
#pragma unroll
      for (int q = 0; q < kC; ++q) n_c += c[q] != 0;
    };
    scan();
    for (int j = 0; j < k; ++j) {
      uint64_t best = c[0];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
        best = o > best ? o : best;
      }
      const int bi = static_cast<int>(~static_cast<uint32_t>(best));
      if (lane == (bi & 31)) {
        elig &= ~(1u << (bi >> 5));
        if (n_c > 1) {
#pragma unroll
          for (int q = 0; q + 1 < kC; ++q) c[q] = c[q + 1];
          c[kC - 1] = 0;
          --n_c;
        } else {
          scan();
        }
      }
      if (lane == j) my_idx = bi;
    }
  }
  __syncwarp();  // the scratch is free for the next token

  // The selected experts' values, recomputed from their logits exactly as the keys were
  // (softmax: the logit; sigmoid: s).
  float my_val = 0.0f;
  if (lane < k) {
    const float l = __ldg(row + my_idx);
    my_val = sigmoid ? sigmoid_keys_f32(l) : l;
  }
  const float top_val = __shfl_sync(0xffffffffu, my_val, 0);

  float g;
  if (sigmoid) {
    g = (lane < k) ? my_val : 0.0f;
    if (renorm) {
      // rank-order sum: lanes 0..k-1 hold the selected s in rank order
      float acc = 0.0f;
      for (int j = 0; j < k; ++j) acc += __shfl_sync(0xffffffffu, g, j);
      g = g / acc;
    }
  } else {
    float num = (lane < k) ? expf(my_val - top_val) : 0.0f;
    float den = 0.0f;
    if (renorm) {
      for (int j = 0; j < k; ++j) den += __shfl_sync(0xffffffffu, num, j);
    } else {
      float part = 0.0f;
#pragma unroll
      for (int i = 0; i < NPL; ++i)
        if (lane + 32 * i < E) part += expf(__ldg(row + lane + 32 * i) - top_val);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      den = part;
    }
    g = num / den;
  }
  if (lane < k) {
    topk_idx[static_cast<size_t>(t) * k + lane] = my_idx;
    topk_w[static_cast<size_t>(t) * k + lane] = g * scale;
  }
}

// One token: its logits, then its selection.
template <int NPL>
__device__ __forceinline__ void route_token(const float* __restrict__ logits,
                                            const float* __restrict__ bias, int t, int E, int k,
                                            int sigmoid, int renorm,
                                            int32_t* __restrict__ topk_idx,
                                            float* __restrict__ topk_w, int lane,
                                            uint8_t* scratch, int n_group = 1,
                                            int topk_group = 1, float scale = 1.0f) {
  float l[NPL];
  route_load<NPL>(logits, t, E, lane, l);
  route_select<NPL>(l, logits, bias, t, E, k, sigmoid, renorm, topk_idx, topk_w, lane, scratch,
                    n_group, topk_group, scale);
}

// Tokens t0, t0 + stride, ... by one warp, the next token's logits loaded while the current
// one is selected (a warp that walks several tokens would otherwise wait out each load).
template <int NPL>
__device__ __forceinline__ void route_tokens(const float* __restrict__ logits,
                                             const float* __restrict__ bias, int t0, int stride,
                                             int T, int E, int k, int sigmoid, int renorm,
                                             int32_t* __restrict__ topk_idx,
                                             float* __restrict__ topk_w, int lane,
                                             uint8_t* scratch, int n_group, int topk_group,
                                             float scale) {
  if (t0 >= T) return;
  float nxt[NPL];
  route_load<NPL>(logits, t0, E, lane, nxt);
  for (int t = t0; t < T; t += stride) {
    float cur[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) cur[i] = nxt[i];
    if (t + stride < T) route_load<NPL>(logits, t + stride, E, lane, nxt);
    route_select<NPL>(cur, logits, bias, t, E, k, sigmoid, renorm, topk_idx, topk_w, lane,
                      scratch, n_group, topk_group, scale);
  }
}


}  // namespace moe
