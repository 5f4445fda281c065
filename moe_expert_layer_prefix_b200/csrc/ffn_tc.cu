// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// linear-1 (+ SwiGLU + requantisation) and linear-2 of every expert, as the source pages'
// pipeline lists them (jiqizhixin, "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了", section
// "Mega MoE 是什么？", pipeline paragraph; FP8 x FP4 paragraph: FP8 activations with FP4
// weights; youleyou, "DeepSeek 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", Tile Kernels
// feature list, quantisation item: FP8 quantisation fused with SwiGLU).
//
// Both GEMMs have the form  D[m, n] = sum_k A[m, k] * B[n, k]  per expert, A = the expert's
// rows of x_perm (or h), B = the expert's K-major weight matrix.  One persistent CTA per SM
// walks a static list of 128 x 256 output tiles (expert, m-block, n-block):
//
//   warp 0      TMA producer: A tile 128 x 128 B and B tile 256 x 128 B per k-step into a
//               4-stage shared-memory ring (128-byte swizzle), completion on an mbarrier
//   warp 1      MMA issuer (one thread): tcgen05.mma 128 x 256 x {16|32} into a TMEM
//               fp32 accumulator (256 columns); tcgen05.commit frees ring stages
//   warp 2      scale-factor producer (block-scaled kinds): writes the UE8M0 scales of the
//               k-step into shared memory in the layout tcgen05.cp expects
//   warps 4..7  epilogue: tcgen05.ld of the accumulator (warp i reads TMEM lanes 32i..32i+31,
//               one output row per thread), SwiGLU + BF16 / E4M3 requantisation (linear-1)
//               or BF16 conversion (linear-2), 16-byte global stores
//
// linear-1 tiles take B rows [n*128, n*128+128) (gate) and [I + n*128, ...) (up), so the
// accumulator holds gate in columns 0..127 and up in 128..255 and each tile yields 128 h
// columns -- exactly one 1x128 requantisation block per row.
//
// Kinds: BF16 x BF16 -> tcgen05.mma kind::f16.  E4M3 x {E4M3, E2M1} -> kind::mxf8f6f4
// block-scaled with one UE8M0 scale per 32 elements of K: the fp32 power-of-two activation
// and E4M3 weight scales convert to UE8M0 losslessly; E2M1 weights carry UE8M0 natively.
// E2M1 tiles are expanded by TMA to one byte per element in shared memory (16U4_ALIGN16B),
// the operand layout kind::mxf8f6f4 reads, while HBM traffic stays at 4 bits per weight.
//
// Every wait is bounded: a stuck pipeline records MOE_ERR_TIMEOUT with its site in the
// device error word, raises a CTA-wide abort flag, drains what it issued, frees TMEM and
// returns.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kRowBytes = 128;          // K bytes per tile row per stage (one swizzle atom)
constexpr int kStages = 4;
constexpr int kATileBytes = kBM * kRowBytes;     // 16 KB
constexpr int kBTileBytes = kBN * kRowBytes;     // 32 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes;
// E2M1 tiles are expanded to one byte per element in shared memory, but the copy's
// transaction count is the packed size (half a byte per element).
constexpr int kStageBytesE2M1 = kATileBytes + kBTileBytes / 2;
constexpr int kSfaBytes = 512;                   // 128 rows x 4 UE8M0
constexpr int kSfbBytes = 1024;                  // 256 rows x 4 UE8M0
constexpr int kTmemCols = 512;
constexpr int kAccCol = 0;
constexpr int kSfaCol = 256;
constexpr int kSfbCol = 260;
constexpr int kThreads = 256;
constexpr int kMaxE = 1024;

struct TcParams {
  const int32_t* offsets;  // [E+1]
  int E, S, K;             // K = reduction length in elements
  int n_tiles;             // n-blocks per m-block
  int w_rows;              // weight rows per expert (2I or H)
  int I;                   // linear-1: offset of the up rows; unused for linear-2
  int n_out;               // output columns (I for linear-1, H for linear-2)
  const float* a_scales;   // fp32 [S, K/128] (block-scaled kinds)
  const void* b_scales;    // E4M3: fp32 [E, w_rows/128, K/128]; E2M1: u8 [E, w_rows, K/32]
  void* out;
  float* out_scales;       // linear-1 with E4M3 h
  int* err;
};

struct SharedState {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int total_tiles;
  int mb_start[kMaxE + 1];  // exclusive prefix of m-blocks per expert
  int offs[kMaxE + 1];
};

struct Tile {
  int e, m0, m_end, nb;
};

__device__ __forceinline__ Tile decode_tile(const SharedState& ss, int E, int n_tiles, int t) {
  const int mb = t / n_tiles;
  Tile tile;
  tile.nb = t - mb * n_tiles;
  int lo = 0, hi = E;  // mb_start[lo] <= mb < mb_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ss.mb_start[mid] <= mb) lo = mid; else hi = mid;
  }
  tile.e = lo;
  tile.m0 = ss.offs[lo] + (mb - ss.mb_start[lo]) * kBM;
  tile.m_end = ss.offs[lo + 1];
  return tile;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

// kBlockScaled: false -> BF16 kind::f16; true -> kind::mxf8f6f4 with A = E4M3 and
// B = E4M3 (kBFmt 0) or E2M1 (kBFmt 5).  kSwiGLU: linear-1 epilogue, else linear-2.
// kOutE4M3: linear-1 stores h as E4M3 + 1x128 scales (else BF16).
template <bool kBlockScaled, int kBFmt, bool kSwiGLU, bool kOutE4M3>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kATileBytes;
  uint8_t* sSF = sB + kStages * kBTileBytes;  // per stage: SFA 512 B then SFB 1024 B
  SharedState& ss = *reinterpret_cast<SharedState*>(sSF + kStages * (kSfaBytes + kSfbBytes));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kElemsPerRow = kBlockScaled ? 128 : 64;  // K elements per stage
  const int KB = p.K / kElemsPerRow;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ss.full[s], kBlockScaled ? 2 : 1);
      mbar_init(&ss.empty[s], 1);
    }
    mbar_init(&ss.acc_full, 1);
    mbar_init(&ss.acc_empty, 4);
    mbar_init(&ss.drain, 1);
    ss.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&ss.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 3) {
    // per-expert m-block prefix (warp-wide chunked scan)
    int carry = 0;
    for (int base = 0; base <= p.E; base += 32) {
      const int e = base + lane;
      int o = 0, cnt = 0;
      if (e <= p.E) {
        o = __ldg(p.offsets + e);
        ss.offs[e] = o;
      }
      if (e < p.E) cnt = (__ldg(p.offsets + e + 1) - o + kBM - 1) / kBM;
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      if (e <= p.E) ss.mb_start[e] = carry + incl - cnt;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    if (lane == 0) ss.total_tiles = ss.mb_start[p.E] * p.n_tiles;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = ss.tmem_base;
  const int total = ss.total_tiles;
  volatile int* abort = &ss.abort;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const Tile tile = decode_tile(ss, p.E, p.n_tiles, t);
        const int brow0 = tile.e * p.w_rows + (kSwiGLU ? tile.nb * 128 : tile.nb * kBN);
        const int brow1 = kSwiGLU ? tile.e * p.w_rows + p.I + tile.nb * 128 : brow0 + 128;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ss.empty[stage], phase ^ 1u, p.err, SITE_GEMM_EMPTY, abort)) break;
          mbar_arrive_expect_tx(&ss.full[stage], kBFmt == 5 ? kStageBytesE2M1 : kStageBytes);
          const int kx = kb * kElemsPerRow;
          tma_load_2d(sA + stage * kATileBytes, &tmA, &ss.full[stage], kx, tile.m0);
          tma_load_2d(sB + stage * kBTileBytes, &tmB, &ss.full[stage], kx, brow0);
          tma_load_2d(sB + stage * kBTileBytes + kBTileBytes / 2, &tmB, &ss.full[stage], kx, brow1);
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort) {
        // drain: wait (bounded) for the copies of the last stages this thread issued
        const int n = issued < kStages ? issued : kStages;
        for (int i = 0; i < n; ++i) {
          if (--stage < 0) {
            stage = kStages - 1;
            phase ^= 1u;
          }
          const long long t0 = clock64();
          while (!mbar_try_wait(&ss.full[stage], phase)) {
            if (clock64() - t0 > kWaitLimitCycles) {
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
      constexpr uint32_t kIdesc = kBlockScaled ? idesc_mxf8f6f4(kBM, kBN, 0u, kBFmt)
                                               : idesc_bf16(kBM, kBN);
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool issued_any = false;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        if (!mbar_wait(&ss.acc_empty, acc_phase ^ 1u, p.err, SITE_GEMM_ACC_EMPTY, abort)) break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ss.full[stage], phase, p.err, SITE_GEMM_FULL, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * kATileBytes);
          const uint32_t b_base = smem_u32(sB + stage * kBTileBytes);
          const uint64_t adesc = desc_kmajor_sw128(a_base);
          const uint64_t bdesc = desc_kmajor_sw128(b_base);
          if constexpr (kBlockScaled) {
            const uint32_t sf = smem_u32(sSF + stage * (kSfaBytes + kSfbBytes));
            tc_cp_32x128b_warpx4(tmem + kSfaCol, desc_sf_32x16(sf));
            tc_cp_32x128b_warpx4(tmem + kSfbCol, desc_sf_32x16(sf + kSfaBytes));
            tc_cp_32x128b_warpx4(tmem + kSfbCol + 4, desc_sf_32x16(sf + kSfaBytes + 512));
          }
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            // advance 32 bytes of K inside the 128-byte swizzle atom
            const uint64_t ad = adesc + static_cast<uint64_t>(ks * 2);
            const uint64_t bd = bdesc + static_cast<uint64_t>(ks * 2);
            const uint32_t acc = (kb | ks) != 0 ? 1u : 0u;
            if constexpr (kBlockScaled) {
              const uint32_t id = kIdesc | (static_cast<uint32_t>(ks) << 4) |
                                  (static_cast<uint32_t>(ks) << 29);
              mma_mxf8f6f4(tmem + kAccCol, ad, bd, id,
                           (tmem + kSfaCol) | (static_cast<uint32_t>(ks) << 30),
                           (tmem + kSfbCol) | (static_cast<uint32_t>(ks) << 30), acc);
            } else {
              mma_bf16(tmem + kAccCol, ad, bd, kIdesc, acc);
            }
          }
          issued_any = true;
          tc_commit(&ss.empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&ss.acc_full);
        acc_phase ^= 1u;
      }
      if (*abort && issued_any) {
        // let the issued MMAs finish before TMEM is released
        tc_commit(&ss.drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(&ss.drain, 0)) {
          if (clock64() - t0 > kWaitLimitCycles) break;
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------------ scale factors
    if constexpr (kBlockScaled) {
      const int KS = p.K / 128;  // fp32 scale columns of A (and of E4M3 B)
      int stage = 0;
      uint32_t phase = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const Tile tile = decode_tile(ss, p.E, p.n_tiles, t);
        const int wr0 = kSwiGLU ? tile.nb * 128 : tile.nb * kBN;      // first B row, atom 0
        const int wr1 = kSwiGLU ? p.I + tile.nb * 128 : wr0 + 128;    // first B row, atom 1
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          // gather this k-step's scale words before waiting for the stage
          uint32_t sfa[4], sfb[8];
#pragma unroll
          for (int r1 = 0; r1 < 4; ++r1) {
            const int m = tile.m0 + lane + 32 * r1;
            const uint32_t b = m < p.S ? ue8m0_of_pow2(__ldg(p.a_scales + static_cast<size_t>(m) * KS + kb))
                                       : 127u;
            sfa[r1] = b * 0x01010101u;
          }
#pragma unroll
          for (int a = 0; a < 2; ++a) {
#pragma unroll
            for (int r1 = 0; r1 < 4; ++r1) {
              int wr = (a == 0 ? wr0 : wr1) + lane + 32 * r1;
              wr = wr < p.w_rows ? wr : p.w_rows - 1;
              uint32_t word;
              if constexpr (kBFmt == 5) {
                const uint8_t* sc = static_cast<const uint8_t*>(p.b_scales) +
                                    (static_cast<size_t>(tile.e) * p.w_rows + wr) * (p.K / 32) + kb * 4;
                word = __ldg(reinterpret_cast<const uint32_t*>(sc));
              } else {
                const float* sc = static_cast<const float*>(p.b_scales) +
                                  (static_cast<size_t>(tile.e) * (p.w_rows / 128) + wr / 128) * KS + kb;
                word = ue8m0_of_pow2(__ldg(sc)) * 0x01010101u;
              }
              sfb[a * 4 + r1] = word;
            }
          }
          if (!mbar_wait(&ss.empty[stage], phase ^ 1u, p.err, SITE_GEMM_SF_EMPTY, abort)) {
            ok = false;
            break;
          }
          uint8_t* sf = sSF + stage * (kSfaBytes + kSfbBytes);
          *reinterpret_cast<uint4*>(sf + 16 * lane) = make_uint4(sfa[0], sfa[1], sfa[2], sfa[3]);
          *reinterpret_cast<uint4*>(sf + kSfaBytes + 16 * lane) =
              make_uint4(sfb[0], sfb[1], sfb[2], sfb[3]);
          *reinterpret_cast<uint4*>(sf + kSfaBytes + 512 + 16 * lane) =
              make_uint4(sfb[4], sfb[5], sfb[6], sfb[7]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ss.full[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp - 4;  // TMEM lane quadrant
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
      const Tile tile = decode_tile(ss, p.E, p.n_tiles, t);
      // every lane waits; the decision is made warp-uniform so that the .sync.aligned
      // TMEM loads below always run with the full warp
      const bool ready = mbar_wait(&ss.acc_full, acc_phase, p.err, SITE_GEMM_ACC_FULL, abort);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const int row = tile.m0 + q * 32 + lane;
      const bool valid = row < tile.m_end;
      if constexpr (kSwiGLU) {
        if constexpr (kOutE4M3) {
          float h[128];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t g[32], u[32];
            tmem_ld32(trow + kAccCol + 32 * c, g);
            tmem_ld32(trow + kAccCol + 128 + 32 * c, u);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              h[32 * c + i] = silu_mul(__uint_as_float(g[i]), __uint_as_float(u[i]));
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ss.acc_empty);
          float amax = 0.0f;
#pragma unroll
          for (int i = 0; i < 128; ++i) amax = fmaxf(amax, fabsf(h[i]));
          const int e = max(e4m3_scale_exponent(amax), -126);
          const float inv = exp2i(-e);
          if (valid) {
            uint8_t* dst = static_cast<uint8_t*>(p.out) + static_cast<size_t>(row) * p.n_out +
                           tile.nb * 128;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int b = 16 * v + 4 * i;
                const __nv_fp8x2_storage_t lo =
                    __nv_cvt_float2_to_fp8x2(make_float2(h[b] * inv, h[b + 1] * inv), __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8x2_storage_t hi =
                    __nv_cvt_float2_to_fp8x2(make_float2(h[b + 2] * inv, h[b + 3] * inv), __NV_SATFINITE, __NV_E4M3);
                w[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
              }
              reinterpret_cast<uint4*>(dst)[v] = make_uint4(w[0], w[1], w[2], w[3]);
            }
            p.out_scales[static_cast<size_t>(row) * (p.n_out / 128) + tile.nb] = exp2i(e);
          }
        } else {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t g[32], u[32];
            tmem_ld32(trow + kAccCol + 32 * c, g);
            tmem_ld32(trow + kAccCol + 128 + 32 * c, u);
            tmem_ld_wait();
            if (valid) {
              uint32_t w[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(
                    silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                    silu_mul(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
                w[i] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                    static_cast<size_t>(row) * p.n_out +
                                                    tile.nb * 128 + 32 * c);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ss.acc_empty);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t d[32];
          tmem_ld32(trow + kAccCol + 32 * c, d);
          tmem_ld_wait();
          const int col = tile.nb * kBN + 32 * c;
          if (valid && col < p.n_out) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const __nv_bfloat162 b2 =
                  __floats2bfloat162_rn(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1]));
              w[i] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                  static_cast<size_t>(row) * p.n_out + col);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ss.acc_empty);
      }
      acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

constexpr size_t kSmemBytes = 1024 /*alignment slack*/ + kStages * kStageBytes +
                              kStages * (kSfaBytes + kSfbBytes) + sizeof(SharedState);

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// 2-D K-major tensor map: rows x K, box {128-byte K slice, 128 rows}, 128-byte swizzle.
// fmt: 0 = BF16, 1 = 8-bit, 2 = E2M1 (expanded to one byte per element in shared memory).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K, int fmt) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  CUtensorMapDataType dt;
  uint64_t row_bytes;
  uint32_t box_k;
  if (fmt == 0) {
    dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    row_bytes = K * 2;
    box_k = 64;
  } else if (fmt == 1) {
    dt = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    row_bytes = K;
    box_k = 128;
  } else {
    dt = CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
    row_bytes = K / 2;
    box_k = 128;
  }
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_k, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kBS, int kBFmt, bool kSw, bool kE4>
cudaError_t launch_tc(const FfnArgs& a, bool linear1, cudaStream_t s) {
  const int K = linear1 ? a.H : a.I;
  const int w_rows = linear1 ? 2 * a.I : a.H;
  CUtensorMap tmA, tmB;
  const int afmt = a.act == MOE_BF16 ? 0 : 1;
  const int bfmt = a.wt == MOE_BF16 ? 0 : (a.wt == MOE_E4M3 ? 1 : 2);
  if (!make_map(&tmA, a.a, static_cast<uint64_t>(a.S), static_cast<uint64_t>(K), afmt))
    return cudaErrorInvalidValue;
  if (!make_map(&tmB, a.w, static_cast<uint64_t>(a.E) * w_rows, static_cast<uint64_t>(K), bfmt))
    return cudaErrorInvalidValue;
  TcParams p;
  p.offsets = a.offsets;
  p.E = a.E;
  p.S = a.S;
  p.K = K;
  p.n_tiles = linear1 ? a.I / 128 : (a.H + kBN - 1) / kBN;
  p.w_rows = w_rows;
  p.I = a.I;
  p.n_out = linear1 ? a.I : a.H;
  p.a_scales = a.a_scales;
  p.b_scales = a.w_scales;
  p.out = a.out;
  p.out_scales = a.out_scales;
  p.err = a.err;
  auto kern = grouped_gemm_tc<kBS, kBFmt, kSw, kE4>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
  if (err != cudaSuccess) return err;
  count_launch();
  kern<<<num_sms(), kThreads, kSmemBytes, s>>>(tmA, tmB, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_linear1_tc(const FfnArgs& a, cudaStream_t s) {
  if (a.E > kMaxE) return cudaErrorNotSupported;
  if (a.act == MOE_BF16 && a.wt == MOE_BF16) return launch_tc<false, 0, true, false>(a, true, s);
  if (a.act == MOE_E4M3 && a.wt == MOE_E4M3) return launch_tc<true, 0, true, true>(a, true, s);
  if (a.act == MOE_E4M3 && a.wt == MOE_E2M1) return launch_tc<true, 5, true, true>(a, true, s);
  return cudaErrorNotSupported;
}

cudaError_t launch_linear2_tc(const FfnArgs& a, cudaStream_t s) {
  if (a.E > kMaxE) return cudaErrorNotSupported;
  if (a.act == MOE_BF16 && a.wt == MOE_BF16) return launch_tc<false, 0, false, false>(a, false, s);
  if (a.act == MOE_E4M3 && a.wt == MOE_E4M3) return launch_tc<true, 0, false, false>(a, false, s);
  if (a.act == MOE_E4M3 && a.wt == MOE_E2M1) return launch_tc<true, 5, false, false>(a, false, s);
  return cudaErrorNotSupported;
}

}  // namespace moe
