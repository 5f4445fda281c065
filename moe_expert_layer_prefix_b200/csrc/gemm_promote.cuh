// Grouped expert GEMMs for E4M3 activations and weights whose fp32 block scales are
// arbitrary (not powers of two), on tcgen05 with per-block promotion.
//
// The layer's scale contract is fp32 per 1x128 activation block and per 128x128 weight block
// (youleyou, "DeepSeek 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", section "Tile
// Kernels：逼近硬件极限的底层优化", feature list, quantisation item: FP8 per-token / per-block
// quantisation; jiqizhixin, "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了", section "Mega MoE
// 是什么？", FP8 x FP4 paragraph).  The block-scaled MMA (gemm_tc.cuh) applies UE8M0 scales,
// i.e. powers of two only.  Here every 128-deep k-step runs plain kind::f8f6f4 MMAs on the
// E4M3 codes into one of two TMEM partial accumulators, and the epilogue warps fold each
// partial into a running fp32 sum in registers with the k-step's scales:
//     acc[r, c] += sa[r, kb] * sb[block(c), kb] * P_kb[r, c]
// which is the definition sum_kb sum_{k in kb} (code_a sa)(code_b sb) up to fp32 rounding.
// The MMA fills partial kb+1 while the epilogue reads partial kb.
//
// Tiles are 128 x 128 (the running sums of 64 columns per thread fit in registers with 8
// epilogue warps).  linear-1 tiles take B rows [64j, 64j + 64) (gate) and [I + 64j, +64) (up)
// and yield 64 h columns; a CTA takes the two tiles of one 128-column h block back to back,
// so that the block's 1x128 E4M3 requantisation sees the whole block.  linear-2 tiles take
// B rows [128j, 128j + 128).
//
// Roles: warp 0 TMA producer (A 16 KB + B 16 KB per stage, 6 stages), warp 1 MMA issuer,
// warps 4..11 epilogue (warp w: TMEM lane quadrant w % 4, column half (w - 4) / 4).  Every
// wait is bounded like the pipeline of gemm_tc.cuh.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace moe {
namespace gemm {

constexpr int kPN = 128;          // accumulator columns of a promotion tile
constexpr int kPStages = 6;
constexpr int kPTileBytes = 16384;  // A (128 rows) and B (128 rows) per stage, 128 B of K each

struct PSmem {
  uint8_t* sA;
  uint8_t* sB;
  SharedState* ss;
};

constexpr size_t kPSmemBytes = 1024 + 2 * kPStages * kPTileBytes + sizeof(SharedState);
static_assert(kPSmemBytes <= 232448, "exceeds the 227 KB of shared memory a CTA may use");

__device__ __forceinline__ PSmem pcarve(uint8_t* smem_raw) {
  PSmem m;
  m.sA = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                    ~static_cast<uintptr_t>(1023));
  m.sB = m.sA + kPStages * kPTileBytes;
  m.ss = reinterpret_cast<SharedState*>(m.sB + kPStages * kPTileBytes);
  return m;
}

__device__ __forceinline__ void pgemm_init(const PSmem& sm) {
  SharedState& ss = *sm.ss;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&ss.full[s], 1);
      mbar_init(&ss.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ss.part_full[b], 1);
      mbar_init(&ss.part_empty[b], kEpiWarps);
    }
    mbar_init(&ss.drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&ss.amax_bar[q], 64);
    ss.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&ss.tmem_base, 256);
    tmem_relinquish();
  }
}

// One grouped GEMM with fp32 block scales.  p.n_tiles counts 128-column tiles (linear-1:
// I / 64, an even number; linear-2: H / 128).  a_scales fp32 [S, K/128]; b_scales fp32
// [E, w_rows/128, K/128].
template <bool kSwiGLU, bool kOutE4M3>
__device__ __forceinline__ void pgemm_phase(const CUtensorMap* tmA_, const CUtensorMap* tmB_,
                                            const TcParams& p, const PSmem& sm) {
  const CUtensorMap& tmA = *tmA_;
  const CUtensorMap& tmB = *tmB_;
  SharedState& ss = *sm.ss;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cid = static_cast<int>(blockIdx.x), ncl = static_cast<int>(gridDim.x);
  const int KB = p.K / 128;
  const int KS = KB;  // fp32 scale columns of A and of B
  // work units: linear-1 takes the two tiles of an h block together
  constexpr int kUnit = kSwiGLU ? 2 : 1;
  const int units = ss.mb_total * p.n_tiles / kUnit;
  const uint32_t tmem = ss.tmem_base;
  volatile int* abort = &ss.abort;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      const uint32_t it0 = it;
      for (int u = cid; u < units && !*abort; u += ncl) {
        for (int sub = 0; sub < kUnit && !*abort; ++sub) {
          const int t = u * kUnit + sub;
          const Tile tile = decode_tile(ss, p.E, p.n_tiles, kBM, t, true);
          const int ebase = tile.e * p.w_rows;
          for (int kb = 0; kb < KB; ++kb) {
            const int stage = static_cast<int>(it % kPStages);
            const uint32_t phase = (it / kPStages) & 1u;
            if (!mbar_wait(&ss.empty[stage], phase ^ 1u, p.err, SITE_GEMM_EMPTY, abort)) break;
            const int kx = kb * 128;
            mbar_arrive_expect_tx(&ss.full[stage], 2 * kPTileBytes);
            tma_load_2d(sm.sA + stage * kPTileBytes, &tmA, &ss.full[stage], kx, tile.m0);
            if constexpr (kSwiGLU) {
              tma_load_2d(sm.sB + stage * kPTileBytes, &tmB, &ss.full[stage], kx,
                          ebase + 64 * tile.nb);
              tma_load_2d(sm.sB + stage * kPTileBytes + kPTileBytes / 2, &tmB, &ss.full[stage],
                          kx, ebase + p.I + 64 * tile.nb);
            } else {
              tma_load_2d(sm.sB + stage * kPTileBytes, &tmB, &ss.full[stage], kx,
                          ebase + kPN * tile.nb);
            }
            ++it;
          }
        }
      }
      if (*abort) {
        // drain: wait (bounded) for the copies of the last stages issued
        const uint32_t issued = it - it0;
        const uint32_t n = issued < static_cast<uint32_t>(kPStages) ? issued : kPStages;
        const long long limit = wait_limit(p.err);
        for (uint32_t i = 1; i <= n; ++i) {
          const int stage = static_cast<int>((it - i) % kPStages);
          const uint32_t phase = ((it - i) / kPStages) & 1u;
          const long long t0 = clock64();
          while (!mbar_try_wait(&ss.full[stage], phase)) {
            if (clock64() - t0 > limit) {
              report_error(p.err, MOE_ERR_TIMEOUT, SITE_GEMM_DRAIN);
              break;
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_f8f6f4_e4m3(kBM, kPN);
      uint32_t it = 0;
      bool issued_any = false;
      bool ok = true;
      for (int u = cid; u < units && ok && !*abort; u += ncl) {
        for (int sub = 0; sub < kUnit && ok; ++sub) {
          for (int kb = 0; kb < KB; ++kb) {
            const int stage = static_cast<int>(it % kPStages);
            const uint32_t b = it & 1u;
            if (!mbar_wait(&ss.full[stage], (it / kPStages) & 1u, p.err, SITE_GEMM_FULL, abort) ||
                !mbar_wait(&ss.part_empty[b], ((it >> 1) & 1u) ^ 1u, p.err, SITE_GEMM_ACC_EMPTY,
                           abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t adesc = desc_kmajor_sw128(smem_u32(sm.sA + stage * kPTileBytes));
            const uint64_t bdesc = desc_kmajor_sw128(smem_u32(sm.sB + stage * kPTileBytes));
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_f8f6f4(tmem + kPN * b, adesc + static_cast<uint64_t>(ks * 2),
                         bdesc + static_cast<uint64_t>(ks * 2), kIdesc, ks != 0 ? 1u : 0u);
            issued_any = true;
            tc_commit(&ss.empty[stage]);
            tc_commit(&ss.part_full[b]);
            ++it;
          }
        }
      }
      if (*abort && issued_any) {
        tc_commit(&ss.drain);
        const long long t0 = clock64();
        const long long limit = wait_limit(p.err);
        while (!mbar_try_wait(&ss.drain, 0)) {
          if (clock64() - t0 > limit) break;
        }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const float* bsc = static_cast<const float*>(p.b_scales);
    const int wblocks = p.w_rows / 128;
    uint32_t it = 0, hq = 0;
    bool ok = true;
    for (int u = cid; u < units && ok && !*abort; u += ncl) {
      float hkeep[32];  // linear-1: the first tile's h values of this thread (E4M3 output)
      for (int sub = 0; sub < kUnit && ok; ++sub) {
        const int t = u * kUnit + sub;
        const Tile tile = decode_tile(ss, p.E, p.n_tiles, kBM, t, true);
        const int row0 = tile.m0 + q * 32;
        const int row = row0 + lane;
        const bool valid = row < tile.m_end;
        const float* sa_row = p.a_scales + static_cast<size_t>(valid ? row : tile.m0) * KS;
        // weight blocks of this thread's columns: linear-1 gate block and up block; linear-2
        // one block (64 of its 128 rows)
        const float* sb0 = bsc + (static_cast<size_t>(tile.e) * wblocks +
                                  (kSwiGLU ? (64 * tile.nb) / 128 : tile.nb)) * KS;
        const float* sb1 = kSwiGLU ? bsc + (static_cast<size_t>(tile.e) * wblocks +
                                            (p.I + 64 * tile.nb) / 128) * KS
                                   : sb0;
        float acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = 0.0f;
        // scales two k-steps ahead of their use (global loads, cached)
        float sa_n = __ldg(sa_row), s0_n = __ldg(sb0), s1_n = __ldg(sb1);
        for (int kb = 0; kb < KB; ++kb) {
          const float sa = sa_n, s0 = s0_n, s1 = s1_n;
          if (kb + 1 < KB) {
            sa_n = __ldg(sa_row + kb + 1);
            s0_n = __ldg(sb0 + kb + 1);
            s1_n = __ldg(sb1 + kb + 1);
          }
          const uint32_t b = it & 1u;
          const bool ready = mbar_wait(&ss.part_full[b], (it >> 1) & 1u, p.err,
                                       SITE_GEMM_ACC_FULL, abort);
          if (!__all_sync(0xffffffffu, ready)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // linear-1: gate columns [32 half, +32) and up columns [64 + 32 half, +32);
          // linear-2: columns [64 half, +64).  Read one 32-column chunk at a time (the
          // running sums and linear-1's kept h values leave no room for both at once).
          const uint32_t c0 = kSwiGLU ? 32u * half : 64u * half;
          const uint32_t c1 = kSwiGLU ? 64u + 32u * half : 64u * half + 32u;
          const float f0 = sa * s0, f1 = sa * s1;
          uint32_t d[32];
          tmem_ld32(trow + kPN * b + c0, d);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = fmaf(__uint_as_float(d[i]), f0, acc[i]);
          tmem_ld32(trow + kPN * b + c1, d);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ss.part_empty[b]);
          ++it;
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[32 + i] = fmaf(__uint_as_float(d[i]), f1, acc[32 + i]);
        }
        if (!ok) break;
        if constexpr (kSwiGLU) {
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) h[i] = silu_mul(acc[i], acc[32 + i]);
          // h columns of this thread: tile t covers [64 nb, +64) of h, this half [32 half, +32)
          const int hcol = 64 * tile.nb + 32 * half;
          if constexpr (kOutE4M3) {
            if (sub == 0) {
#pragma unroll
              for (int i = 0; i < 32; ++i) hkeep[i] = h[i];
              continue;
            }
            // second tile of the h block: amax over both tiles' 64 values of this thread,
            // then over the other column half (the exponent exchange of gemm_tc.cuh)
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fmaxf(fabsf(h[i]), fabsf(hkeep[i])));
            constexpr int kNoExp = -128;
            const int own = amax > 0.0f ? max(e4m3_scale_exponent(amax), -126) : kNoExp;
            const int slot = static_cast<int>(hq & 1u);
            ss.ecode[slot][half][q * 32 + lane] = static_cast<int8_t>(own);
            mbar_arrive(&ss.amax_bar[q]);
            const bool got = mbar_wait(&ss.amax_bar[q], hq & 1u, p.err, SITE_GEMM_AMAX, abort);
            ++hq;
            if (!__all_sync(0xffffffffu, got)) {
              ok = false;
              break;
            }
            const int both = max(own, static_cast<int>(ss.ecode[slot][half ^ 1][q * 32 + lane]));
            const int e = both == kNoExp ? 0 : both;
            const float inv = exp2i(-e);
            if (valid) {
              uint8_t* base = static_cast<uint8_t*>(p.out) + static_cast<size_t>(row) * p.n_out;
#pragma unroll
              for (int part = 0; part < 2; ++part) {
                const float* src = part == 0 ? hkeep : h;
                uint8_t* dst = base + hcol - 64 + 64 * part;
#pragma unroll
                for (int v = 0; v < 2; ++v) {
                  uint32_t w[4];
#pragma unroll
                  for (int i = 0; i < 4; ++i) {
                    const int bb = 16 * v + 4 * i;
                    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                        make_float2(src[bb] * inv, src[bb + 1] * inv), __NV_SATFINITE, __NV_E4M3);
                    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                        make_float2(src[bb + 2] * inv, src[bb + 3] * inv), __NV_SATFINITE, __NV_E4M3);
                    w[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
                  }
                  reinterpret_cast<uint4*>(dst)[v] = make_uint4(w[0], w[1], w[2], w[3]);
                }
              }
              if (half == 0)
                p.out_scales[static_cast<size_t>(row) * (p.n_out / 128) + (64 * tile.nb) / 128] =
                    exp2i(e);
            }
          } else {
            if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                    static_cast<size_t>(row) * p.n_out + hcol);
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const __nv_bfloat162 b2 =
                      __floats2bfloat162_rn(h[8 * v + 2 * i], h[8 * v + 2 * i + 1]);
                  w[i] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        } else {
          // y columns [128 nb + 64 half, +64) of the warp's 32 rows, BF16
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          const int rows_ok = min(32, tile.m_end - row0);
          const int chunks_ok = min(8, (p.n_out - kPN * tile.nb - 64 * half) / 8);
          store_rows_coalesced<8>(
              w, reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(p.out) +
                                            static_cast<size_t>(row0) * p.n_out +
                                            kPN * tile.nb + 64 * half),
              static_cast<size_t>(p.n_out) * 2, rows_ok, chunks_ok, lane);
        }
      }
    }
  }
}

}  // namespace gemm
}  // namespace moe
