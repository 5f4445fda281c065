// Grouped expert GEMM kernel (gemm_tc.cuh holds the tensor-core pipeline and its source)
// and its host-side launchers: tensor maps, tile-shape choice, cluster launch.
#include "common.cuh"
#include "gemm_promote.cuh"
#include "gemm_tc.cuh"
#include "internal.h"

namespace moe {

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

// 2-D K-major tensor map: rows x K, box {128-byte K slice, box_rows rows}, 128-byte swizzle.
// fmt: 0 = BF16, 1 = 8-bit, 2 = E2M1 (expanded to one byte per element in shared memory).
bool make_kmajor_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K, int fmt,
                     uint32_t box_rows) {
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
  const cuuint32_t box[2] = {box_k, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


namespace {

using namespace gemm;

template <int kCta, int kTm, bool kBlockScaled, int kBFmt, bool kSwiGLU, bool kOutE4M3,
          bool kDGate>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const Smem sm = carve<kCta, kTm>(smem_raw);
  gemm_init<kCta, kBlockScaled, kTm>(sm, &tmA, 1);
  if (threadIdx.x == 0) tma_prefetch_desc(&tmB);
  gemm_prefix<kCta, kTm>(sm, p.offsets, p.E);
  tc_fence_before();
  __syncthreads();
  if constexpr (kCta == 2) cluster_sync();  // the peer's barriers exist before anyone signals them
  tc_fence_after();
  Pipe pipe;
  gemm_phase<kCta, kBlockScaled, kBFmt, kSwiGLU, kOutE4M3, kTm, kDGate>(&tmA, &tmB, p, sm, pipe);
  tc_fence_before();
  __syncthreads();
  // in a pair, neither CTA leaves while the other may still touch its shared memory
  if constexpr (kCta == 2) cluster_sync();
  tc_fence_after();
  gemm_fini<kCta>(sm);
}

// E4M3 x E4M3 with arbitrary fp32 block scales (gemm_promote.cuh).
template <bool kSwiGLU, bool kOutE4M3>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_promote(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, const TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const PSmem sm = pcarve(smem_raw);
  pgemm_init(sm);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  const Smem list{sm.sA, sm.sB, nullptr, sm.ss};
  gemm_prefix<1, kBM>(list, p.offsets, p.E);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pgemm_phase<kSwiGLU, kOutE4M3>(&tmA, &tmB, p, sm);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if ((threadIdx.x >> 5) == 1) {
    __syncwarp();
    tmem_dealloc(sm.ss->tmem_base, 256);
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
template <int kCta, int kTm, bool kBS, int kBFmt, bool kSw, bool kE4, bool kDG = false>
cudaError_t launch_tc(const FfnArgs& a, bool linear1, cudaStream_t s) {
  const int K = linear1 ? a.H : a.I;
  const int w_rows = linear1 ? 2 * a.I : a.H;
  CUtensorMap tmA, tmB;
  const int afmt = a.act == MOE_BF16 ? 0 : 1;
  const int bfmt = a.wt == MOE_BF16 ? 0 : (a.wt == MOE_E4M3 ? 1 : 2);
  if (!make_kmajor_map(&tmA, a.a, static_cast<uint64_t>(a.S), static_cast<uint64_t>(K), afmt, kTm))
    return cudaErrorInvalidValue;
  if (!make_kmajor_map(&tmB, a.w, static_cast<uint64_t>(a.E) * w_rows, static_cast<uint64_t>(K), bfmt))
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
  p.dh = a.dh;
  p.err = a.err;
  auto kern = grouped_gemm_tc<kCta, kTm, kBS, kBFmt, kSw, kE4, kDG>;
  const size_t smem = Cfg<kCta, kTm>::kSmem;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((num_sms() / kCta) * kCta);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCta;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, p);
}

template <bool kSw, bool kE4>
cudaError_t launch_promote(const FfnArgs& a, bool linear1, cudaStream_t s) {
  const int K = linear1 ? a.H : a.I;
  const int w_rows = linear1 ? 2 * a.I : a.H;
  CUtensorMap tmA, tmB;
  if (!make_kmajor_map(&tmA, a.a, static_cast<uint64_t>(a.S), static_cast<uint64_t>(K), 1, 128))
    return cudaErrorInvalidValue;
  // linear-1 loads the gate and the up half of a tile as two 64-row boxes
  if (!make_kmajor_map(&tmB, a.w, static_cast<uint64_t>(a.E) * w_rows, static_cast<uint64_t>(K), 1,
                       linear1 ? 64 : 128))
    return cudaErrorInvalidValue;
  TcParams p{};
  p.offsets = a.offsets;
  p.E = a.E;
  p.S = a.S;
  p.K = K;
  p.n_tiles = linear1 ? a.I / 64 : a.H / 128;
  p.w_rows = w_rows;
  p.I = a.I;
  p.n_out = linear1 ? a.I : a.H;
  p.a_scales = a.a_scales;
  p.b_scales = a.w_scales;
  p.out = a.out;
  p.out_scales = a.out_scales;
  p.err = a.err;
  auto kern = grouped_gemm_promote<kSw, kE4>;
  const size_t smem = kPSmemBytes;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  count_launch();
  kern<<<num_sms(), kThreads, smem, s>>>(tmA, tmB, p);
  return cudaGetLastError();
}

template <bool kBS, int kBFmt, bool kSw, bool kE4, bool kDG = false>
cudaError_t launch_tc_any(const FfnArgs& a, bool linear1, cudaStream_t s) {
  switch (gemm_tile_shape(a.act, a.S, a.E, true)) {
    case 2: return launch_tc<2, kBM, kBS, kBFmt, kSw, kE4, kDG>(a, linear1, s);
    case 3: return launch_tc<1, 32, kBS, kBFmt, kSw, kE4, kDG>(a, linear1, s);
    default: return launch_tc<1, kBM, kBS, kBFmt, kSw, kE4, kDG>(a, linear1, s);
  }
}

}  // namespace

// Tile shape.  Pairs (M = 256) once the average expert holds at least 128 rows, for BF16:
// block-scaled pairs are correct but slower than single CTAs (the per-SM k-step rate is the
// same and the 256-row tiles carry more padding).  Small tiles (32-row m-blocks) when the
// average expert holds at most 16 rows, as in decode: the weights stream from HBM once per
// m-block either way, and the smaller A box leaves room for a fifth pipeline stage.
// Single CTAs (M = 128) otherwise.
int gemm_tile_shape(int act, int S, int E, bool allow_pair) {
  int mode = gemm_tile_mode();
  if (mode == 2 && !allow_pair) mode = 1;
  if (mode == 1) return 1;
  if (mode == 2) return num_sms() >= 2 ? 2 : 1;
  if (mode == 3) return 3;
  if (static_cast<int64_t>(S) <= 16LL * E) return 3;
  if (allow_pair && act == MOE_BF16 && static_cast<int64_t>(S) >= 128LL * E && num_sms() >= 2)
    return 2;
  return 1;
}

cudaError_t launch_linear1_tc(const FfnArgs& a, cudaStream_t s) {
  if (a.E > kMaxE) return cudaErrorNotSupported;
  if (a.scale_fmt == MOE_SCALE_FP32) {
    if (a.act != MOE_E4M3 || a.wt != MOE_E4M3) return cudaErrorNotSupported;
    return launch_promote<true, true>(a, true, s);
  }
  if (a.act == MOE_BF16 && a.wt == MOE_BF16) return launch_tc_any<false, 0, true, false>(a, true, s);
  if (a.act == MOE_E4M3 && a.wt == MOE_E4M3) return launch_tc_any<true, 0, true, true>(a, true, s);
  if (a.act == MOE_E4M3 && a.wt == MOE_E2M1) return launch_tc_any<true, 5, true, true>(a, true, s);
  return cudaErrorNotSupported;
}

cudaError_t launch_linear1_dgate_tc(const FfnArgs& a, cudaStream_t s) {
  if (a.E > kMaxE) return cudaErrorNotSupported;
  if (a.act != MOE_BF16 || a.wt != MOE_BF16 || a.dh == nullptr) return cudaErrorNotSupported;
  return launch_tc_any<false, 0, true, false, true>(a, true, s);
}

cudaError_t launch_linear2_tc(const FfnArgs& a, cudaStream_t s) {
  if (a.E > kMaxE) return cudaErrorNotSupported;
  if (a.scale_fmt == MOE_SCALE_FP32) {
    if (a.act != MOE_E4M3 || a.wt != MOE_E4M3) return cudaErrorNotSupported;
    return launch_promote<false, false>(a, false, s);
  }
  if (a.act == MOE_BF16 && a.wt == MOE_BF16) return launch_tc_any<false, 0, false, false>(a, false, s);
  if (a.act == MOE_E4M3 && a.wt == MOE_E4M3) return launch_tc_any<true, 0, false, false>(a, false, s);
  if (a.act == MOE_E4M3 && a.wt == MOE_E2M1) return launch_tc_any<true, 5, false, false>(a, false, s);
  return cudaErrorNotSupported;
}

}  // namespace moe
