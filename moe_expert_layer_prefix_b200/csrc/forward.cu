// The whole MoE layer in one persistent launch: route -> dispatch -> linear-1 + SwiGLU +
// requant -> linear-2 -> combine.
//
// This is the "mega-kernel" of the source pages: dispatch, both linear layers, SwiGLU and
// combine fused into one kernel instead of one launch per step (jiqizhixin,
// "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了", section "Mega MoE 是什么？", the mega-kernel
// paragraph; the routing step in front of it follows youleyou, "DeepSeek 模型更新解读 Tile
// Kernels 与 DeepEP V2 新特性", Tile Kernels feature list, gating item).  On one GPU there is
// no communication to overlap; what the fusion removes is the launch gaps and the host
// round trips between the steps.
//
// One CTA per SM, all co-resident (cooperative launch).  Phases are separated by grid-wide
// barriers with bounded waits; each phase runs exactly the device code of the standalone
// kernels (route.cuh, dispatch.cuh, gemm_tc.cuh, combine.cuh), so moe_forward produces the
// same bytes as the unfused chain of entry points.  Data produced by one phase is read by the
// next through L2 (ld.global.cg), and the phases whose output a TMA copy reads (x_perm, h)
// end with a generic-to-async proxy fence.  The shared memory of the GEMM ring doubles as
// the dispatch phases' scratch (chunk masks, slot tables, offsets), and one TMEM
// allocation serves both GEMM phases, whose pipeline counters carry over.
#include "combine.cuh"
#include "common.cuh"
#include "dispatch.cuh"
#include "gemm_tc.cuh"
#include "internal.h"
#include "route.cuh"

namespace moe {
namespace {

using namespace gemm;

struct FwdParams {
  const void* x;
  const float* x_scales;
  const float* logits;
  const float* bias;
  int sigmoid, renorm, T, H, E, k, C;
  int row_bytes;
  int quant_x;  // x is BF16 and the dispatch quantises it to E4M3 + 1x128 scales
  int n_group, topk_group;
  float scale;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* offsets;
  int32_t* perm_src;
  int32_t* slot_of;
  void* x_perm;
  float* x_perm_scales;
  int32_t* cnt;
  int32_t* totals;
  void* y;
  void* out;
  uint32_t* bar;
  int* err;
  TcParams l1, l2;
};

// kCta = 2: the GEMM phases run on CTA pairs (cta_group::2, M = 256 tiles); the launch is
// then a cluster launch of pairs, and every other phase treats the CTAs as before.
template <bool kBS, int kBFmt, bool kE4, int kTm, int kCta>
__global__ void __launch_bounds__(kThreads, 1)
moe_forward_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW1,
                   const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW2,
                   const FwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const Smem sm = carve<kCta, kTm>(smem_raw);
  gemm_init<kCta, kBS, kTm>(sm, &tmX, 1);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmH);
    tma_prefetch_desc(&tmW2);
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kCta == 2) cluster_sync();  // the peer's barriers exist before anyone signals them
  tc_fence_after();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = kThreads / 32;
  const int gw = blockIdx.x * nwarps + warp, GW = gridDim.x * nwarps;
  // dispatch scratch inside the (idle) GEMM ring, which is at least 180 KB: per-warp chunk
  // masks (8 x E words, at most 32 KB), then scan partials, offsets and warp sums
  uint8_t* scratch = sm.sA;
  uint32_t* mask = reinterpret_cast<uint32_t*>(scratch) + warp * p.E;
  int32_t(*part)[33] = reinterpret_cast<int32_t(*)[33]>(scratch + nwarps * kMaxE * 4);
  int32_t* soffs = reinterpret_cast<int32_t*>(scratch + nwarps * kMaxE * 4 + 32 * 33 * 4);
  int32_t* wsum = soffs + 1028;

  // A grid barrier that timed out (recorded in the error word) ends the phases for this
  // CTA: it releases TMEM and returns; the other CTAs give up at their next barrier.
  do {
    // 1. route: one warp per token, candidate scratch per warp in the idle GEMM ring
    uint8_t* rscr = scratch + warp * kRouteScratchBytes;
    if (p.E <= 256)
      route_tokens<8>(p.logits, p.bias, gw, GW, p.T, p.E, p.k, p.sigmoid, p.renorm, p.topk_idx,
                      p.topk_w, lane, rscr, p.n_group, p.topk_group, p.scale);
    else
      route_tokens<32>(p.logits, p.bias, gw, GW, p.T, p.E, p.k, p.sigmoid, p.renorm, p.topk_idx,
                       p.topk_w, lane, rscr, p.n_group, p.topk_group, p.scale);
    if (!grid_sync(p.bar, p.err)) break;

    // 2. per-chunk expert counts
    for (int c = gw; c < p.C; c += GW) hist_chunk(mask, p.topk_idx, p.T, p.E, p.k, c, lane, p.cnt);
    if (!grid_sync(p.bar, p.err)) break;

    // 3. per-expert scans over the chunks (32 experts per CTA pass)
    for (int g = blockIdx.x; g < (p.E + 31) / 32; g += gridDim.x)
      scan_group(p.cnt, p.E, p.C, p.totals, g, nwarps, warp, lane, part);
    if (!grid_sync(p.bar, p.err)) break;

    // 4. expert offsets (every CTA keeps its own copy; CTA 0 publishes them)
    offsets_from_totals(p.totals, p.E, soffs, wsum);
    if (blockIdx.x == 0)
      for (int e = threadIdx.x; e <= p.E; e += blockDim.x) p.offsets[e] = soffs[e];

    // 5. slots and permutation (one warp per 32-token chunk)
    for (int c = gw; c < p.C; c += GW)
      assign_slots_chunk(mask, p.topk_idx, p.T, p.E, p.k, c, p.cnt, soffs, p.perm_src, p.slot_of,
                         lane);
    if (!grid_sync(p.bar, p.err)) break;

    // 6. row copies x -> x_perm (one warp per token), quantising BF16 rows when asked
    if (p.quant_x) {
      for (int t = gw; t < p.T; t += GW)
        quant_copy_token_rows(static_cast<const __nv_bfloat16*>(p.x), p.H, p.slot_of, t, p.k,
                              static_cast<uint8_t*>(p.x_perm), p.x_perm_scales, lane);
    } else {
      for (int t = gw; t < p.T; t += GW)
        copy_token_rows(static_cast<const uint8_t*>(p.x), p.x_scales, p.row_bytes, p.H / 128,
                        p.slot_of, t, p.k, static_cast<uint8_t*>(p.x_perm), p.x_perm_scales, lane);
    }
    fence_proxy_async_global();  // x_perm is read by TMA next
    if (!grid_sync(p.bar, p.err)) break;

    // 7. linear-1 + SwiGLU + requantisation.  The m-block list is computed once for both
    //    GEMMs (the same offsets and tile shape).
    Pipe pipe;
    gemm_prefix<kCta, kTm>(sm, p.offsets, p.E);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    gemm_phase<kCta, kBS, kBFmt, true, kE4, kTm>(&tmX, &tmW1, p.l1, sm, pipe);
    fence_proxy_async_global();  // h is read by TMA next
    if (!grid_sync(p.bar, p.err)) break;

    // 8. linear-2
    gemm_phase<kCta, kBS, kBFmt, false, false, kTm>(&tmH, &tmW2, p.l2, sm, pipe);
    if (!grid_sync(p.bar, p.err)) break;

    // 9. combine.  A warp keeps two 16-byte loads per lane and source row in flight and
    //    takes a whole token when there are tokens enough for every warp; fewer tokens are
    //    split into 512-column chunks.
    if (p.T >= 2 * GW) {
      for (int t = gw; t < p.T; t += GW)
        combine_token<false, 2>(p.y, p.slot_of, p.topk_w, t, p.k, p.H, p.out, lane, 0, p.H / 8);
    } else {
      const int nc = combine_chunks<2>(p.H);
      const int width = nc == 1 ? p.H / 8 : 64;
      const long items = static_cast<long>(p.T) * nc;
      for (long it = gw; it < items; it += GW) {
        const int t = static_cast<int>(it / nc), c = static_cast<int>(it % nc);
        combine_token<false, 2>(p.y, p.slot_of, p.topk_w, t, p.k, p.H, p.out, lane, c * width,
                                (c + 1) * width);
      }
    }
  } while (0);

  tc_fence_before();
  __syncthreads();
  // in a pair, neither CTA leaves while the other may still touch its shared memory
  if constexpr (kCta == 2) cluster_sync();
  tc_fence_after();
  gemm_fini<kCta>(sm);
}

template <bool kBS, int kBFmt, bool kE4, int kTm, int kCta>
cudaError_t launch(const ForwardArgs& a, cudaStream_t s) {
  const int S = a.T * a.k;
  const int afmt = a.act == MOE_BF16 ? 0 : 1;
  const int bfmt = a.wt == MOE_BF16 ? 0 : (a.wt == MOE_E4M3 ? 1 : 2);
  CUtensorMap tmX, tmW1, tmH, tmW2;
  if (!make_kmajor_map(&tmX, a.x_perm, S, a.H, afmt, kTm) ||
      !make_kmajor_map(&tmW1, a.w1, static_cast<uint64_t>(a.E) * 2 * a.I, a.H, bfmt) ||
      !make_kmajor_map(&tmH, a.h, S, a.I, afmt, kTm) ||
      !make_kmajor_map(&tmW2, a.w2, static_cast<uint64_t>(a.E) * a.H, a.I, bfmt))
    return cudaErrorInvalidValue;
  FwdParams p;
  p.x = a.x;
  p.x_scales = a.x_scales;
  p.logits = a.logits;
  p.bias = a.bias;
  p.sigmoid = a.sigmoid;
  p.renorm = a.renorm;
  p.n_group = a.n_group;
  p.topk_group = a.topk_group;
  p.scale = a.scale;
  p.T = a.T;
  p.H = a.H;
  p.E = a.E;
  p.k = a.k;
  p.C = (a.T + kChunkTokens - 1) / kChunkTokens;
  p.row_bytes = a.H * (a.act == MOE_BF16 ? 2 : 1);
  p.quant_x = a.act == MOE_E4M3 && a.x_scales == nullptr;
  p.topk_idx = a.topk_idx;
  p.topk_w = a.topk_w;
  p.offsets = a.offsets;
  p.perm_src = a.perm_src;
  p.slot_of = a.slot_of;
  p.x_perm = a.x_perm;
  p.x_perm_scales = a.x_perm_scales;
  p.cnt = a.cnt;
  p.totals = a.totals;
  p.y = a.y;
  p.out = a.out;
  p.bar = a.bar;
  p.err = a.err;
  TcParams l1{}, l2{};
  l1.offsets = l2.offsets = a.offsets;
  l1.E = l2.E = a.E;
  l1.S = l2.S = S;
  l1.I = l2.I = a.I;
  l1.err = l2.err = a.err;
  l1.K = a.H;
  l1.n_tiles = a.I / 128;
  l1.w_rows = 2 * a.I;
  l1.n_out = a.I;
  l1.a_scales = a.x_perm_scales;
  l1.b_scales = a.w1_scales;
  l1.out = a.h;
  l1.out_scales = a.h_scales;
  l2.K = a.I;
  l2.n_tiles = (a.H + kBN - 1) / kBN;
  l2.w_rows = a.H;
  l2.n_out = a.H;
  l2.a_scales = a.h_scales;
  l2.b_scales = a.w2_scales;
  l2.out = a.y;
  l2.out_scales = nullptr;
  p.l1 = l1;
  p.l2 = l2;

  auto kern = moe_forward_kernel<kBS, kBFmt, kE4, kTm, kCta>;
  const size_t smem = Cfg<kCta, kTm>::kSmem;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if constexpr (kCta == 2) {
    // pairs: as many clusters as can be resident at once (every CTA waits at the grid
    // barriers, so all of them must be), at most one CTA per SM
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t q = cfg;
    q.attrs = attr + 1;
    q.numAttrs = 1;
    int clusters = 0;
    err = cudaOccupancyMaxActiveClusters(&clusters, kern, &q);
    if (err != cudaSuccess) return err;
    clusters = min(clusters, num_sms() / 2);
    if (clusters < 1) return cudaErrorNotSupported;
    cfg.gridDim = dim3(2 * clusters);
    cfg.numAttrs = 2;
  }
  err = cudaMemsetAsync(a.bar, 0, 2 * sizeof(uint32_t), s);
  if (err != cudaSuccess) return err;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kern, tmX, tmW1, tmH, tmW2, p);
}

}  // namespace

cudaError_t launch_forward_fused(const ForwardArgs& a, cudaStream_t s) {
  // the dispatch phases keep per-warp masks (8 x E words) in the idle GEMM ring
  if (a.E > 1024) return cudaErrorNotSupported;
  // the chain's tile choice (1 single, 2 pair, 3 small), so that both compute the same bytes
  const int shape = gemm_tile_shape(a.act, a.T * a.k, a.E, true);
  if (a.act == MOE_BF16 && a.wt == MOE_BF16)
    return shape == 3   ? launch<false, 0, false, 32, 1>(a, s)
           : shape == 2 ? launch<false, 0, false, kBM, 2>(a, s)
                        : launch<false, 0, false, kBM, 1>(a, s);
  if (a.act == MOE_E4M3 && a.wt == MOE_E4M3)
    return shape == 3   ? launch<true, 0, true, 32, 1>(a, s)
           : shape == 2 ? launch<true, 0, true, kBM, 2>(a, s)
                        : launch<true, 0, true, kBM, 1>(a, s);
  if (a.act == MOE_E4M3 && a.wt == MOE_E2M1)
    return shape == 3   ? launch<true, 5, true, 32, 1>(a, s)
           : shape == 2 ? launch<true, 5, true, kBM, 2>(a, s)
                        : launch<true, 5, true, kBM, 1>(a, s);
  return cudaErrorNotSupported;
}

}  // namespace moe
