// Weight gradients of the BF16 expert layer on the 5th-generation tensor cores.
//
//   dW1_e = dG_e^T x_e   [2I, H],     dW2_e = dy_w,e^T h_e   [H, I]     (fp32)
//
// (youleyou, "DeepSeek 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", section "Tile
// Kernels：逼近硬件极限的底层优化", feature list: the batched-transpose item and the
// model-layer item, wrappers that make the kernels trainable layers.)
//
// The reduction runs over an expert's slots, which are the rows of the slot-major operands.
// tcgen05 reads K-major tiles, so each operand is first transposed into an expert-padded
// copy Xt [C, Kp]: expert e's slots occupy columns [pk_e, pk_e + n_e) and are followed by
// zeros up to the next multiple of 64, pk_e = sum over f < e of roundup(n_f, 64).  Every
// 64-deep k-step of a tile then lies inside one expert's segment, starts on a 128-byte
// boundary (as TMA needs), and the padding columns multiply zeros.
//
// The GEMM: one CTA per SM walks tiles (expert, 128-row m-block, 256-column n-block);
// warp 0 loads A (128 x 64) and B (256 x 64) tiles with TMA into a 4-stage ring, warp 1
// issues tcgen05.mma kind::f16 into a TMEM fp32 accumulator, warps 4..11 read it out (two
// per TMEM lane quadrant, 128 columns each) and store fp32 rows.  Experts without slots get
// zero gradients.  Bounded waits as in the forward GEMM.
#include "common.cuh"
#include "gemm_tc.cuh"
#include "internal.h"

namespace moe {
namespace {

using namespace gemm;

constexpr int kWK = 64;          // K elements (BF16) per k-step: 128 bytes
constexpr int kWStages = 4;
constexpr int kWATile = 128 * 128;   // bytes: 128 rows x 128 B
constexpr int kWBTile = 256 * 128;   // bytes: 256 rows x 128 B

// padded segment starts: pk[e] = sum_{f<e} roundup(offsets[f+1] - offsets[f], 64), pk[E]
// the total (one block, E <= 1024)
__global__ void __launch_bounds__(1024) pad_offsets_kernel(const int32_t* __restrict__ offsets,
                                                            int E, int32_t* __restrict__ pk) {
  __shared__ int32_t part[1024];
  const int e = threadIdx.x;
  const int n = e < E ? __ldg(offsets + e + 1) - __ldg(offsets + e) : 0;
  part[e] = (n + kWK - 1) / kWK * kWK;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {  // inclusive scan (Hillis-Steele)
    const int v = e >= o ? part[e - o] : 0;
    __syncthreads();
    part[e] += v;
    __syncthreads();
  }
  if (e < E) pk[e + 1] = part[e];
  if (e == 0) pk[0] = 0;
}

// Xt[c][pk_e + i] = X[offsets[e] + i][c] (i < n_e), 0 for n_e <= i < roundup(n_e, 64).
// 32 x 32 tiles through shared memory; blocks past pk[E] return.
__global__ void __launch_bounds__(256) pad_transpose_kernel(
    const uint16_t* __restrict__ X, int C, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ pk, int E, int Kp, uint16_t* __restrict__ Xt) {
  __shared__ uint16_t tile[32][34];
  const int k0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  if (k0 >= __ldg(pk + E)) return;
  int lo = 0, hi = E;  // pk[lo] <= k0 < pk[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(pk + mid) <= k0) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int a = __ldg(offsets + e), n = __ldg(offsets + e + 1) - a;
  const int i0 = k0 - __ldg(pk + e);
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
  for (int r = ty; r < 32; r += 8) {
    const int i = i0 + r, c = c0 + tx;
    tile[r][tx] = (i < n && c < C) ? X[static_cast<size_t>(a + i) * C + c] : uint16_t(0);
  }
  __syncthreads();
#pragma unroll
  for (int r = ty; r < 32; r += 8) {
    const int c = c0 + r;
    if (c < C) Xt[static_cast<size_t>(c) * Kp + k0 + tx] = tile[tx][r];
  }
}

struct WgParams {
  const int32_t* offsets;  // [E+1]
  const int32_t* pk;       // [E+1] padded segment starts
  int E, M, N;             // out[e] is M x N
  int m_tiles, n_tiles;    // M / 128, ceil(N / 256)
  float* out;
  int* err;
};

struct WgShared {
  uint64_t full[kWStages];
  uint64_t empty[kWStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__global__ void __launch_bounds__(kThreads, 1)
wgrad_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const WgParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sA = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sB = sA + kWStages * kWATile;
  WgShared& ss = *reinterpret_cast<WgShared*>(sB + kWStages * kWBTile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kWStages; ++s) {
      mbar_init(&ss.full[s], 1);
      mbar_init(&ss.empty[s], 1);
    }
    mbar_init(&ss.acc_full, 1);
    mbar_init(&ss.acc_empty, kEpiWarps);
    mbar_init(&ss.drain, 1);
    ss.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&ss.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ss.tmem_base;
  volatile int* abort = &ss.abort;
  const int tpe = p.m_tiles * p.n_tiles;  // tiles per expert
  const int total = p.E * tpe;
  // tile t: expert t / tpe, m-block (t % tpe) / n_tiles, n-block (t % tpe) % n_tiles
  auto k_steps = [&](int e) {
    return (__ldg(p.offsets + e + 1) - __ldg(p.offsets + e) + kWK - 1) / kWK;
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const int e = t / tpe, r = t % tpe, mb = r / p.n_tiles, nb = r % p.n_tiles;
        const int KB = k_steps(e);
        const int kx0 = __ldg(p.pk + e);
        for (int kb = 0; kb < KB; ++kb) {
          const int stage = static_cast<int>(it % kWStages);
          if (!mbar_wait(&ss.empty[stage], ((it / kWStages) & 1u) ^ 1u, p.err, SITE_GEMM_EMPTY,
                         abort))
            break;
          mbar_arrive_expect_tx(&ss.full[stage], kWATile + kWBTile);
          const int kx = kx0 + kb * kWK;
          tma_load_2d(sA + stage * kWATile, &tmA, &ss.full[stage], kx, 128 * mb);
          tma_load_2d(sB + stage * kWBTile, &tmB, &ss.full[stage], kx, 256 * nb);
          tma_load_2d(sB + stage * kWBTile + kWBTile / 2, &tmB, &ss.full[stage], kx,
                      256 * nb + 128);
          ++it;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16(kBM, kBN);
      uint32_t it = 0, tiles = 0;
      bool issued_any = false;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const int KB = k_steps(t / tpe);
        if (KB == 0) continue;  // the epilogue stores zeros for an expert without slots
        if (!mbar_wait(&ss.acc_empty, (tiles & 1u) ^ 1u, p.err, SITE_GEMM_ACC_EMPTY, abort)) break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          const int stage = static_cast<int>(it % kWStages);
          if (!mbar_wait(&ss.full[stage], (it / kWStages) & 1u, p.err, SITE_GEMM_FULL, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = desc_kmajor_sw128(smem_u32(sA + stage * kWATile));
          const uint64_t bd = desc_kmajor_sw128(smem_u32(sB + stage * kWBTile));
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)  // 16 BF16 of K per MMA: 32 bytes inside the atom
            mma_bf16(tmem, ad + static_cast<uint64_t>(ks * 2), bd + static_cast<uint64_t>(ks * 2),
                     kIdesc, (kb | ks) != 0 ? 1u : 0u);
          issued_any = true;
          tc_commit(&ss.empty[stage]);
          ++it;
        }
        if (!ok) break;
        tc_commit(&ss.acc_full);
        ++tiles;
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
    const int q = warp & 3, half = (warp - 4) >> 2;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t tiles = 0;
    for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
      const int e = t / tpe, r = t % tpe, mb = r / p.n_tiles, nb = r % p.n_tiles;
      const int row0 = 128 * mb + 32 * q;
      const int col0 = 256 * nb + 128 * half;
      const int chunks_ok = min(32, (p.N - col0) / 4);  // 16-byte chunks (4 fp32) in range
      float* orow0 = p.out + (static_cast<size_t>(e) * p.M + row0) * p.N + col0;
      uint32_t w[128];
      if (k_steps(e) == 0) {
#pragma unroll
        for (int i = 0; i < 128; ++i) w[i] = 0u;
      } else {
        const bool ready = mbar_wait(&ss.acc_full, tiles & 1u, p.err, SITE_GEMM_ACC_FULL, abort);
        if (!__all_sync(0xffffffffu, ready)) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(trow + 128 * half + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(w + 32 * c));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ss.acc_empty);
        ++tiles;
      }
      if (chunks_ok > 0)
        store_rows_coalesced<32>(w, reinterpret_cast<uint8_t*>(orow0),
                                 static_cast<size_t>(p.N) * 4, 32, chunks_ok, lane);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 256);
  }
}

constexpr size_t kWgSmem = 1024 + kWStages * (kWATile + kWBTile) + sizeof(WgShared);
static_assert(kWgSmem <= 232448, "exceeds the 227 KB of shared memory a CTA may use");

}  // namespace

size_t wgrad_pad_cols(int S, int E) { return (static_cast<size_t>(S) + 64 * static_cast<size_t>(E) + 63) / 64 * 64; }

cudaError_t launch_wgrad_pad_offsets(const int32_t* offsets, int E, int32_t* pk, cudaStream_t s) {
  count_launch();
  pad_offsets_kernel<<<1, 1024, 0, s>>>(offsets, E, pk);
  return cudaGetLastError();
}

cudaError_t launch_pad_transpose(const void* X, int S, int C, const int32_t* offsets,
                                 const int32_t* pk, int E, void* Xt, cudaStream_t s) {
  const int Kp = static_cast<int>(wgrad_pad_cols(S, E));
  const dim3 grid((C + 31) / 32, Kp / 32);
  count_launch();
  pad_transpose_kernel<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(X), C, offsets, pk, E, Kp,
                                            static_cast<uint16_t*>(Xt));
  return cudaGetLastError();
}

// out[e] [M, N] fp32 = At[:, seg_e] . Bt[:, seg_e]^T with At [M, Kp], Bt [N, Kp] BF16 from
// launch_pad_transpose (M a multiple of 128, N of 128).
cudaError_t launch_wgrad_tc(const void* At, const void* Bt, const int32_t* offsets,
                            const int32_t* pk, int S, int E, int M, int N, float* out, int* err,
                            cudaStream_t s) {
  const uint64_t Kp = wgrad_pad_cols(S, E);
  CUtensorMap tmA, tmB;
  if (!make_kmajor_map(&tmA, At, static_cast<uint64_t>(M), Kp, 0, 128) ||
      !make_kmajor_map(&tmB, Bt, static_cast<uint64_t>(N), Kp, 0, 128))
    return cudaErrorInvalidValue;
  WgParams p;
  p.offsets = offsets;
  p.pk = pk;
  p.E = E;
  p.M = M;
  p.N = N;
  p.m_tiles = M / 128;
  p.n_tiles = (N + 255) / 256;
  p.out = out;
  p.err = err;
  cudaError_t e = cudaFuncSetAttribute(wgrad_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kWgSmem));
  if (e != cudaSuccess) return e;
  count_launch();
  wgrad_tc_kernel<<<num_sms(), kThreads, kWgSmem, s>>>(tmA, tmB, p);
  return cudaGetLastError();
}

}  // namespace moe
