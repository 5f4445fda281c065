// Device helpers shared by the library's kernels: error reporting, bounded waits and thin
// inline-PTX wrappers for the sm_100a features the kernels use (mbarrier, TMA,
// tcgen05 / TMEM).  Nothing here computes any part of the MoE layer itself.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// ---------------------------------------------------------------------------------------
// device error word: err[0] = moe_status, err[1] = site; the first failure wins
// ---------------------------------------------------------------------------------------
enum Site : int {
  SITE_GEMM_FULL = 101,      // MMA issuer waiting for a filled smem stage
  SITE_GEMM_EMPTY = 102,     // loader waiting for a free smem stage
  SITE_GEMM_ACC_FULL = 103,  // epilogue waiting for a finished accumulator
  SITE_GEMM_ACC_EMPTY = 104, // MMA issuer waiting for the epilogue to drain TMEM
  SITE_GEMM_SF_EMPTY = 105,  // scale-factor loader waiting for a free smem stage
  SITE_GEMM_DRAIN = 106,     // loader draining its in-flight copies after an abort
  SITE_GEMM_AMAX = 107,      // linear-1 epilogue waiting for the other half's row amax
  SITE_GRID_BARRIER = 201,   // persistent kernel waiting at a grid-wide barrier
  SITE_SCALE_FORMAT = 301,   // an fp32 block scale that is not a positive normal power of two
  SITE_SELFTEST_MBAR = 901,  // self-test: a wait on an mbarrier nothing ever arrives on
};

__device__ __forceinline__ void report_error(int* err, int code, int site) {
  if (err != nullptr && atomicCAS(err, 0, code) == 0) atomicExch(err + 1, site);
}

// The device control block the error pointer of every waiting kernel points at:
// {status, site, wait limit in SM clock cycles (64-bit, 8-byte aligned)}.  The limit is
// process-wide per device (moe_set_wait_limit); about one second at the B200's boost clock
// by default, while legitimate waits are microseconds.
constexpr long long kWaitLimitCycles = 2000000000LL;

__device__ __forceinline__ long long wait_limit(const int* err) {
  if (err == nullptr) return kWaitLimitCycles;
  const long long v = *reinterpret_cast<const volatile long long*>(err + 2);
  return v > 0 ? v : kWaitLimitCycles;
}

// ---------------------------------------------------------------------------------------
// small utilities
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .b32 r;\n\t.reg .pred p;\n\t"
      "elect.sync r|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(pred));
  return pred != 0;
}

// ---------------------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

template <bool kCluster>
__device__ __forceinline__ bool mbar_try_wait_scoped(uint64_t* bar, uint32_t parity) {
  if constexpr (kCluster) return mbar_try_wait_cluster(bar, parity);
  else return mbar_try_wait(bar, parity);
}

// Waits until the phase with parity `parity` of `bar` has completed.  Gives up after
// kWaitLimitCycles (or at once if *abort is set by another role), records the failure in
// the error word, raises *abort and returns false.
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err, int site,
                                          volatile int* abort) {
  if (mbar_try_wait_scoped<kCluster>(bar, parity)) return true;
  const long long t0 = clock64();
  const long long limit = wait_limit(err);
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_scoped<kCluster>(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (clock64() - t0 > limit) {
        report_error(err, MOE_ERR_TIMEOUT, site);
        *abort = 1;
        return false;
      }
    }
  }
}

// A counter in shared memory published by one warp (release) and polled by another
// (acquire): the hand-off from the GEMM's stager warp to its MMA-issuing thread.
__device__ __forceinline__ void st_release_shared(uint32_t* p, uint32_t v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_shared(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}

// Polls the counter until it reaches `target` and returns the value seen (0 when it gave
// up); bounded like mbar_wait (gives up after the wait limit or once *abort is raised,
// recording MOE_ERR_TIMEOUT at SITE_GEMM_FULL).  A caller that keeps the returned value
// needs no poll at all for the k-steps it already covers.
__device__ __forceinline__ uint32_t wait_ready(const uint32_t* p, uint32_t target, int* err,
                                               volatile int* abort) {
  uint32_t v = ld_acquire_shared(p);
  if (v >= target) return v;
  const long long t0 = clock64();
  const long long limit = wait_limit(err);
  for (uint32_t it = 1;; ++it) {
    v = ld_acquire_shared(p);
    if (v >= target) return v;
    if ((it & 255u) == 0) {
      if (*abort) return 0;
      if (clock64() - t0 > limit) {
        report_error(err, MOE_ERR_TIMEOUT, SITE_GEMM_FULL);
        *abort = 1;
        return 0;
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// clusters (CTA pairs for cta_group::2 tensor-core tiles)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of all CTAs in the cluster (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// shared::cluster address of the variable at local shared address `saddr` in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// Arrive on an mbarrier given by its shared::cluster address (possibly in the peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// ---------------------------------------------------------------------------------------
// TMA (no multicast anywhere in this library)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Pair form: the destination is this CTA's shared memory, the completion goes to the
// mbarrier at shared::cluster address `bar_cluster` (the pair leader's).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}

// Orders this thread's generic-proxy global writes before later async-proxy (TMA) reads.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later async-proxy
// (TMA / tcgen05) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Asynchronous 4-byte global -> shared copy (the copy engine of cp.async: nothing waits on
// the data in registers).  Source and destination must be 4-byte aligned.
__device__ __forceinline__ void cp_async_4(void* dst_smem, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src)
               : "memory");
}

// Asynchronous 16-byte global -> shared copy (cached in L2 only).  Both addresses must be
// 16-byte aligned.
__device__ __forceinline__ void cp_async_16(void* dst_smem, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src)
               : "memory");
}

// One arrival on bar once every cp.async this thread has issued so far has landed; the
// barrier's expected count must include it (.noinc).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// ---------------------------------------------------------------------------------------
// tcgen05 / TMEM
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major operand tile stored by TMA with 128-byte
// swizzling: 8-row x 128-byte swizzle atoms, consecutive atoms 1024 bytes apart.
// Fields: start address >> 4 [0,14), leading byte offset >> 4 [16,30) (unused for swizzled
// K-major tiles), stride byte offset >> 4 [32,46), version 1 [46,48), layout [61,64).
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(16u >> 4) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
  return d;
}

// Descriptor of an unswizzled source of tcgen05.cp 32x128b: 32 rows of 16 bytes, stored
// contiguously, i.e. four 8x16-byte core matrices 128 bytes apart along the rows.
__device__ __forceinline__ uint64_t desc_sf_32x16(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(0) << 16;
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;  // layout 0 = no swizzle
}

// Instruction descriptor, kind::f16 with BF16 A/B, FP32 accumulator, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor, kind::f8f6f4 (no block scaling), E4M3 A and B, FP32 accumulator,
// both K-major.
__host__ __device__ constexpr uint32_t idesc_f8f6f4_e4m3(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f8f6f4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Instruction descriptor, kind::mxf8f6f4 block-scaled, UE8M0 scales, both K-major.
// Format codes: E4M3 = 0, E2M1 = 5.  The scale-factor byte selectors (bits [4,6) for B and
// [29,31) for A) are OR-ed in per MMA.
__host__ __device__ constexpr uint32_t idesc_mxf8f6f4(int M, int N, uint32_t afmt, uint32_t bfmt) {
  return (afmt << 7) | (bfmt << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_mxf8f6f4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t tmem_sfa,
                                             uint32_t tmem_sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::
          "r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tmem_sfa), "r"(tmem_sfb));
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_mxf8f6f4_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                                  uint32_t idesc, uint32_t tmem_sfa,
                                                  uint32_t tmem_sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::
          "r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tmem_sfa), "r"(tmem_sfb));
}

// Pair form of tc_commit: arrives on the mbarrier at the same shared offset in every CTA
// of `cta_mask` (tcgen05.commit with the cluster multicast form; no TMA is involved).
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

__device__ __forceinline__ void tc_cp_32x128b_warpx4_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Arrives (once) on `bar` when all previously issued tcgen05 operations of this thread
// have completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Copies a 32-row x 128-bit shared-memory matrix into TMEM lanes [0,32) of each of the four
// 32-lane sub-partitions (four 32-bit columns starting at taddr).
__device__ __forceinline__ void tc_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------------------
// number formats used by the kernels
// ---------------------------------------------------------------------------------------
// UE8M0 byte of a positive power-of-two fp32 scale (its biased exponent field).
__device__ __forceinline__ uint32_t ue8m0_of_pow2(float s) {
  return (__float_as_uint(s) >> 23) & 0xFFu;
}

// Nonzero when the fp32 bit pattern w is not a positive normal power of two (sign or
// mantissa bits set, zero / subnormal or Inf / NaN exponent field): such a scale has no
// exact UE8M0 byte.
__device__ __forceinline__ uint32_t not_pow2_scale(uint32_t w) {
  const uint32_t e = (w >> 23) & 0xFFu;
  return (w & 0x807FFFFFu) | static_cast<uint32_t>(e == 0u || e == 0xFFu);
}

// Smallest n with a <= 448 * 2^n for a > 0 finite (448 = 1.75 * 2^8).  With
// a = m * 2^ea, 1 <= m < 2: n = ea - 8 if m <= 1.75, else ea - 7.  Subnormal a is handled
// by normalising first.  Returns 0 for a == 0.
__device__ __forceinline__ int e4m3_scale_exponent(float a) {
  if (!(a > 0.0f)) return 0;
  uint32_t b = __float_as_uint(a);
  int ea = static_cast<int>((b >> 23) & 0xFF);
  uint32_t mant = b & 0x7FFFFFu;
  if (ea == 0) {  // subnormal: normalise the mantissa
    int sh = __clz(mant) - 8;
    mant = (mant << sh) & 0x7FFFFFu;
    ea = 1 - sh;
  }
  ea -= 127;
  // m <= 1.75  <=>  mantissa field <= 0.75 * 2^23
  return (mant <= 0x600000u) ? ea - 8 : ea - 7;
}

__device__ __forceinline__ float exp2i(int n) {  // 2^n for -126 <= n <= 127
  return __uint_as_float(static_cast<uint32_t>(n + 127) << 23);
}

// ---------------------------------------------------------------------------------------
// grid-wide barrier for co-resident (cooperative) grids: bar[0] arrivals, bar[1] generation
// (both zero before the launch).  `expected` arrivals complete it (the grid's CTA count).
// Bounded: gives up after the wait limit, records MOE_ERR_TIMEOUT at SITE_GRID_BARRIER and
// returns false (in every thread of the CTA).
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ bool grid_sync(uint32_t* bar, int* err, uint32_t expected) {
  __syncthreads();
  int ok = 1;  // thread 0's result, shared through the closing barrier (no shared memory)
  if (threadIdx.x == 0) {
    const uint32_t gen = ld_acquire_gpu(bar + 1);
    __threadfence();
    const uint32_t arrived = atomicAdd(bar, 1u);
    if (arrived == expected - 1) {
      atomicExch(bar, 0u);
      __threadfence();
      atomicAdd(bar + 1, 1u);
    } else {
      const long long t0 = clock64();
      const long long limit = wait_limit(err);
      while (ld_acquire_gpu(bar + 1) == gen) {
        if (clock64() - t0 > limit) {
          report_error(err, MOE_ERR_TIMEOUT, SITE_GRID_BARRIER);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
  }
  return __syncthreads_and(ok) != 0;
}

__device__ __forceinline__ bool grid_sync(uint32_t* bar, int* err) {
  return grid_sync(bar, err, gridDim.x);
}

}  // namespace moe
