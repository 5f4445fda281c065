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

// (key, id) ordering: larger key first, then lower id.
__device__ __forceinline__ bool better(float ka, int ia, float kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

// One warp selects the k experts of token t and writes topk_idx[t, :], topk_w[t, :].
// Lanes hold experts lane, lane+32, ...; all 32 lanes must call it together.
// Group-limited selection (n_group > 1, groups of G = E / n_group experts with G a multiple
// of 32): a group's score is the fp32 sum of its two largest keys, the topk_group best groups
// (equal scores -> lower group) are kept and the k experts are chosen among theirs only.
// Gates are multiplied by `scale` (the routed scaling factor).  n_group = 1, scale = 1 is
// the plain router.
template <int NPL>  // experts per lane (E <= 32 * NPL)
__device__ __forceinline__ void route_token(const float* __restrict__ logits,
                                            const float* __restrict__ bias, int t, int E, int k,
                                            int sigmoid, int renorm,
                                            int32_t* __restrict__ topk_idx,
                                            float* __restrict__ topk_w, int lane,
                                            int n_group = 1, int topk_group = 1,
                                            float scale = 1.0f) {
  const float* row = logits + static_cast<size_t>(t) * E;

  float key[NPL];
  float val[NPL];  // softmax: the logit; sigmoid: s
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const float l = __ldg(row + e);
      if (sigmoid) {
        const float s = sigmoid_keys_f32(l);
        val[i] = s;
        key[i] = __fadd_rn(s, bias ? __ldg(bias + e) : 0.0f);
      } else {
        val[i] = l;
        key[i] = l;
      }
    } else {
      val[i] = 0.0f;
      key[i] = -INFINITY;
    }
  }

  // Selection.  A candidate is packed into one 64-bit word ordered like (key, id): the key
  // as an order-preserving integer in the high half (-0 taken as +0, so that equal keys give
  // equal words), the complemented id in the low half (lower id wins a tie).  0 is below
  // every candidate.  Each lane caches its best four untaken candidates; a round takes the
  // warp maximum of the lanes' best (5 shuffle steps), the winning lane moves its list up,
  // and only a lane whose four are all taken rescans its NPL experts.
  auto pack = [](float key, int e) -> uint64_t {
    uint32_t u = __float_as_uint(__fadd_rn(key, 0.0f));
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (static_cast<uint64_t>(u) << 32) | static_cast<uint32_t>(~e);
  };
  // Groups.  Lane l holds experts l + 32i, so with G a multiple of 32 a group is sg = G / 32
  // consecutive slots i of every lane: each lane keeps a running top-2 over the group's
  // slots and the warp merges them at the group's last slot; slots of groups that are not
  // kept start out as taken.
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
  // This lane's best four untaken candidates in order (c[0] best; 0 = none) and their
  // values; the winning lane shifts its list up and rescans only once all four are gone.
  constexpr int kC = 4;
  uint64_t c[kC];
  float cv[kC];
  int n_c = 0;  // valid entries of c
  auto scan = [&]() {
#pragma unroll
    for (int q = 0; q < kC; ++q) {
      c[q] = 0;
      cv[q] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u)) {
        const uint64_t x = pack(key[i], e);
        if (x > c[kC - 1]) {  // insert, keeping c sorted
          uint64_t y = x;
          float yv = val[i];
#pragma unroll
          for (int q = 0; q < kC; ++q) {
            if (y > c[q]) {
              const uint64_t t0 = c[q];
              const float tv = cv[q];
              c[q] = y;
              cv[q] = yv;
              y = t0;
              yv = tv;
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
  int my_idx = 0;      // lane j keeps the j-th selection
  float my_val = 0.0f;
  float top_val = 0.0f;
  for (int j = 0; j < k; ++j) {
    uint64_t best = c[0];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
      best = o > best ? o : best;
    }
    const int bi = static_cast<int>(~static_cast<uint32_t>(best));
    const int owner = bi & 31;
    const float bv = __shfl_sync(0xffffffffu, cv[0], owner);
    if (lane == owner) {
      taken |= 1u << (bi >> 5);
      if (n_c > 1) {
#pragma unroll
        for (int q = 0; q + 1 < kC; ++q) {
          c[q] = c[q + 1];
          cv[q] = cv[q + 1];
        }
        c[kC - 1] = 0;
        --n_c;
      } else {
        scan();
      }
    }
    if (lane == j) {
      my_idx = bi;
      my_val = bv;
    }
    if (j == 0) top_val = bv;
  }

  float g;
  if (sigmoid) {
    g = (lane < k) ? my_val : 0.0f;
    if (renorm) {
      float sum = g;
      // rank-order sum: lanes 0..k-1 hold the selected s in rank order
      float acc = 0.0f;
      for (int j = 0; j < k; ++j) acc += __shfl_sync(0xffffffffu, sum, j);
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
        if (lane + 32 * i < E) part += expf(val[i] - top_val);
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


}  // namespace moe
