// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// linear-1 (+ SwiGLU + requantisation) and linear-2 of every expert, as the source pages'
// pipeline lists them (jiqizhixin, "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了", section
// "Mega MoE 是什么？", pipeline paragraph; FP8 x FP4 paragraph: FP8 activations with FP4
// weights; youleyou, "DeepSeek 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", Tile Kernels
// feature list, quantisation item: FP8 quantisation fused with SwiGLU).
//
// Both GEMMs have the form  D[m, n] = sum_k A[m, k] * B[n, k]  per expert, A = the expert's
// rows of x_perm (or h), B = the expert's K-major weight matrix.  Persistent CTAs (one per
// SM) walk a static list of output tiles (expert, m-block, n-block) of N = 256 columns
// (decode_tile gives its order).
// Tile shapes (Cfg below):
//   single  one CTA, M = 128: A 128 x 128 B and B 256 x 128 B per k-step, 4 stages
//   small   one CTA, 32-row m-blocks: a 32-row A box, 5 stages
//   pair    a 2-CTA cluster, M = 256 (tcgen05 cta_group::2): each CTA loads its own 128 A
//           rows and half of the B rows (128 x 128 B) per k-step, 6 stages; the leader CTA
//           issues the MMAs, which read both CTAs' shared memory and write both CTAs' TMEM,
//           so each weight tile crosses L2 -> SM once per 256 rows and each SM moves 32 KB
//           per k-step instead of 48 KB.
// Roles per CTA:
//   warp 0      TMA producer into the shared-memory ring (128-byte swizzle); in a pair, both
//               CTAs' copies complete on the leader's stage barrier
//   warp 1      MMA issuer (one thread, leader CTA): tcgen05.mma 128|256 x 256 x {16|32}
//               into a TMEM fp32 accumulator (256 columns); tcgen05.commit frees ring stages
//               (in both CTAs of a pair).  It waits on the stage barriers itself, except for
//               E2M1 weights over K loops of 8 or more k-steps: there it polls a shared-
//               memory count of ready k-steps that the stager publishes (an mbarrier wait
//               costs the issuing thread about as much as the four MMAs of a k-step, and
//               E2M1 adds two scale copies per k-step on the same thread)
//   warp 2      scale loader (block-scaled kinds): copies the raw scales of each group of 4
//               k-steps into a 4-slot shared-memory ring with asynchronous copies (cp.async)
//   warp 3      scale converter (block-scaled kinds): UE8M0 bytes in the layout tcgen05.cp
//               reads, one barrier arrival per group; as the stager (see warp 1) it also
//               waits for each k-step's A/B stage and publishes the ready count; before each
//               GEMM phase it also builds the tile list
//   warps 4..11 epilogue: two warps per TMEM lane quadrant (warp w reads lanes
//               32(w%4)..+31, one output row per thread), each taking half of the tile's
//               columns, so that the accumulator is read out in a quarter of the time and
//               handed back to the MMA issuer before any arithmetic: SwiGLU + BF16 / E4M3
//               requantisation (linear-1; the two halves of a row exchange their partial
//               amax through shared memory), or in the backward form of linear-1 the
//               gradients of gate and up from dh, or BF16 conversion (linear-2); 16-byte
//               global stores, for linear-2 after lane pairs swap chunks so that every store
//               writes whole 32-byte sectors
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
// Shared by the grouped-GEMM kernel and the persistent forward kernel.  Every wait is
// bounded: a stuck pipeline records MOE_ERR_TIMEOUT with its site in the
// device error word, raises a CTA-wide abort flag, drains what it issued, frees TMEM and
// returns.
#pragma once

#include "common.cuh"

namespace moe {
namespace gemm {

constexpr int kBM = 128;           // accumulator rows per CTA (TMEM lanes)
constexpr int kBN = 256;           // accumulator columns (MMA N)
constexpr int kRowBytes = 128;     // K bytes per tile row per stage (one swizzle atom)
constexpr int kTmemCols = 512;
constexpr int kAccCol = 0;
constexpr int kSfaCol = 256;       // scale-factor column sets start here ...
constexpr int kSfbCol = 260;       // ... SFA (4 columns) then SFB (8 columns)
constexpr int kSfSetCols = 12;
constexpr int kSfSets = 4;         // rotated (per copy) so that a copy never overwrites the
                                   // scales an earlier k-step's MMAs may still be reading
constexpr int kEpiWarps = 8;       // two warps per TMEM lane quadrant, one per column half
constexpr int kThreads = 32 * (4 + kEpiWarps);
constexpr int kMaxE = 1024;
constexpr int kMaxStages = 6;
// Scale-factor ring: one slot per group of 4 k-steps (16 k-steps ahead of the MMA issuer),
// decoupled from the A/B ring.  Slot layout (bytes):
//   [0, 2048)     A: the raw fp32 scales of the CTA's 128 rows, 16 B (4 k-steps) per row,
//                 rewritten in place into 32 lines x 16 B of UE8M0 (line l, word c = row
//                 32c + l, byte j = k-step j of the group) -- the 32x128b layout tcgen05.cp reads
//   [2048, 6144)  B, E2M1: the raw UE8M0 bytes of the tile's 256 rows, 16 B per row (4 k-steps
//                 x 4 sub-blocks of 32), rewritten in place into 4 k-steps x 2 atoms x 512 B
//   [2048, 3072)  B, E4M3: 2 atoms x 512 B of UE8M0 (every row of an atom carries the scale
//                 of its 128-row weight block); the raw fp32 block scales at [3072, 3104)
constexpr int kSfGroups = 4;
constexpr int kSfSlotBytes = 6144;
constexpr int kSfBOff = 2048;
constexpr int kSfBRawE4 = 3072;

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
  const void* dh;          // linear-1 backward form (kDGate): the gradient of h, BF16 [S, I]
  int* err;
};

struct SharedState {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t sf_raw[kSfGroups];   // loader -> converter: raw scale words staged in the slot
  uint64_t sf_full[kSfGroups];  // converters -> MMA issuer: slot converted (one per CTA)
  uint64_t sf_empty[kSfGroups]; // MMA issuer -> loaders: slot copied to TMEM and consumed
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint64_t part_full[2];        // fp32-scale path: partial accumulator b written by the MMAs
  uint64_t part_empty[2];       // ... and read out by every epilogue warp
  uint64_t amax_bar[4];         // linear-1 E4M3 epilogue: both column halves of a quadrant
                                // have published their row's scale exponent
  int8_t ecode[2][2][kBM];      // [tile parity][column half][row of the tile]: the scale
                                // exponent of the half's amax (kNoExp for an all-zero half)
  uint32_t tmem_base;
  int abort;
  int mb_total;             // m-blocks over all experts (tiles = mb_total x n-blocks)
  uint32_t ready;           // stager -> MMA issuer: k-steps whose A/B stage (and scales) are
                            // in shared memory, counted over the whole launch
  int mb_start[kMaxE + 1];  // exclusive prefix of m-blocks per expert
  int offs[kMaxE + 1];
};

// Tile shapes: kCta CTAs per tile, kTm rows of the tile per CTA.  (1, 128) single,
// (2, 128) pair, (1, 32) small: 32-row m-blocks for decode-sized batches, whose A box is a
// quarter of the single one, which buys a fifth stage.  The MMA keeps M = 128: rows past
// kTm read whatever the neighbouring stage holds and their outputs are never stored.
template <int kCta, int kTm = kBM>
struct Cfg {
  static_assert(kTm == kBM || (kCta == 1 && kTm == 32), "unsupported tile shape");
  static constexpr int kStages = kCta == 2 ? 6 : (kTm == kBM ? 4 : 5);
  static_assert(kStages <= kMaxStages, "the stage barriers would overlap the next ones");
  static constexpr int kATileBytes = kTm * kRowBytes;     // 16 KB (4 KB small)
  static constexpr int kBRows = kBN / kCta;               // B rows this CTA loads per k-step
  static constexpr int kBTileBytes = kBRows * kRowBytes;  // 32 KB single, 16 KB pair
  static constexpr int kTileM = kTm * kCta;               // rows of one tile
  static constexpr size_t kSmem = 1024 + kStages * (kATileBytes + kBTileBytes) +
                                  kSfGroups * kSfSlotBytes + sizeof(SharedState);
  static_assert(kSmem <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
};

struct Tile {
  int e, m0, m_end, nb;
};

// Tile t of the list: expert e owns tiles [mb_start[e], mb_start[e + 1]) x n_tiles, numbered
// n-block-major inside the expert (all of its m-blocks for n-block 0, then n-block 1, ...),
// so that the CTAs working side by side on an expert with several m-blocks share each weight
// tile while it is in L2 instead of reading it again a wave later.  mb_major numbers them
// m-block-major instead (consecutive tiles: the n-blocks of one m-block).
__device__ __forceinline__ Tile decode_tile(const SharedState& ss, int E, int n_tiles, int tile_m,
                                            int t, bool mb_major = false) {
  const int q = t / n_tiles;  // in [mb_start[e], mb_start[e + 1]) exactly for e's tiles
  int lo = 0, hi = E;  // mb_start[lo] <= q < mb_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ss.mb_start[mid] <= q) lo = mid; else hi = mid;
  }
  Tile tile;
  tile.e = lo;
  int mb;  // the m-block inside the expert
  if (mb_major) {
    // (no second division: this sits on the issuing threads' path once per tile, and the
    // tiles of short K loops are only a few k-steps long)
    mb = q - ss.mb_start[lo];
    tile.nb = t - q * n_tiles;
  } else {
    const int nmb = ss.mb_start[lo + 1] - ss.mb_start[lo];
    const int local = t - ss.mb_start[lo] * n_tiles;
    tile.nb = local / nmb;
    mb = local - tile.nb * nmb;
  }
  tile.m0 = ss.offs[lo] + mb * tile_m;
  tile.m_end = ss.offs[lo + 1];
  return tile;
}

// silu(g) * u = g * u / (1 + e^-g) with the fast exponential and division (a few ulp; far
// below the BF16 / E4M3 storage step of h).  For g -> -inf the quotient goes to 0.
__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g * u, 1.0f + __expf(-g));
}

// Epilogue stores of linear-2.  Each epilogue thread owns one output row (its TMEM lane), so
// stores straight from registers write 16 bytes into each of 32 rows per warp instruction:
// half sectors, which the memory system takes far more slowly than whole ones (linear-2's
// 512-byte rows of y made the whole GEMM up to 40 % slower).  Instead each pair of lanes
// swaps halves of kEpiGroup x kEpiGroup blocks of 16-byte chunks with shuffles (one butterfly
// stage per doubling of kEpiGroup), after which store instruction j of a group writes
// 16 * kEpiGroup contiguous bytes of the group's row j: whole 32-byte sectors for pairs.
// (Groups of 4 measured the same, groups of 8 slower: the shuffles share the issue path with
// the pipeline's barrier traffic.  linear-1's 128-byte h rows keep the direct stores, which
// measured faster there.)
constexpr int kEpiGroup = 2;

// w holds the thread's row as 16-byte chunks (chunk c = words 4c..4c+3); block kB is chunks
// kEpiGroup*kB .. +kEpiGroup-1.  Afterwards thread i of its group holds, in chunk slot
// kEpiGroup*kB + j, the chunk kEpiGroup*kB + i of the group's row j.
template <int kB, int kN>
__device__ __forceinline__ void transpose_block(uint32_t (&w)[kN], int lane) {
#pragma unroll
  for (int k = 1; k < kEpiGroup; k <<= 1) {
    const bool upper = (lane & k) != 0;
#pragma unroll
    for (int j = 0; j < kEpiGroup; ++j) {
      if (j & k) continue;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint32_t& lo = w[4 * (kEpiGroup * kB + j) + v];
        uint32_t& hi = w[4 * (kEpiGroup * kB + (j ^ k)) + v];
        const uint32_t y = __shfl_xor_sync(0xffffffffu, upper ? lo : hi, k);
        if (upper) lo = y;
        else hi = y;
      }
    }
  }
}

template <int kB, int kBlocks, int kN>
__device__ __forceinline__ void store_blocks(uint32_t (&w)[kN], uint8_t* lane_base, size_t pitch,
                                             int rows_left, int chunks_left, int lane) {
  if constexpr (kB < kBlocks) {
    transpose_block<kB>(w, lane);
#pragma unroll
    for (int j = 0; j < kEpiGroup; ++j) {
      if (j < rows_left && kEpiGroup * kB < chunks_left)
        *reinterpret_cast<uint4*>(lane_base + j * pitch + 16 * kEpiGroup * kB) =
            make_uint4(w[4 * (kEpiGroup * kB + j)], w[4 * (kEpiGroup * kB + j) + 1],
                       w[4 * (kEpiGroup * kB + j) + 2], w[4 * (kEpiGroup * kB + j) + 3]);
    }
    store_blocks<kB + 1, kBlocks>(w, lane_base, pitch, rows_left, chunks_left, lane);
  }
}

// Stores the warp's 32 rows of kChunks 16-byte chunks.  row0 points at the warp's first row
// (lane 0's), pitch is the row pitch in bytes, rows_ok the number of leading rows of the warp
// that exist, chunks_ok the number of leading chunks inside the output (both warp-uniform).
template <int kChunks>
__device__ __forceinline__ void store_rows_coalesced(uint32_t (&w)[4 * kChunks], uint8_t* row0,
                                                     size_t pitch, int rows_ok, int chunks_ok,
                                                     int lane) {
  static_assert(kChunks % kEpiGroup == 0, "chunks come in whole blocks");
  const int g = lane / kEpiGroup, i = lane % kEpiGroup;
  // this lane writes rows kEpiGroup*g + j and chunks kEpiGroup*b + i
  uint8_t* lane_base = row0 + static_cast<size_t>(kEpiGroup * g) * pitch + 16 * i;
  store_blocks<0, kChunks / kEpiGroup>(w, lane_base, pitch, rows_ok - kEpiGroup * g,
                                       chunks_ok - i, lane);
}

// Per-thread pipeline counters.  Each role advances only its own; they carry over from one
// GEMM phase to the next inside a kernel so that the mbarrier phase parities stay in step.
struct Pipe {
  uint32_t prod_it = 0;  // producer: k-steps issued into the ring
  uint32_t mma_it = 0;   // MMA issuer: k-steps consumed
  uint32_t tiles = 0;    // MMA issuer / epilogue: accumulator uses
  uint32_t sf_it = 0;    // scale loader / converter: groups of 4 k-steps staged
  uint32_t sf_grp = 0;   // MMA issuer: groups of 4 k-steps whose scales were copied to TMEM
  uint32_t hq = 0;       // epilogue: linear-1 tiles requantised to E4M3 (amax exchanges)
  uint32_t st_it = 0;    // stager: k-steps published as ready
};

// Shared-memory carve-up (1024-byte aligned; identical offsets in both CTAs of a pair).
struct Smem {
  uint8_t* sA;
  uint8_t* sB;
  uint8_t* sSF;
  SharedState* ss;
};

template <int kCta, int kTm = kBM>
__device__ __forceinline__ Smem carve(uint8_t* smem_raw) {
  using C = Cfg<kCta, kTm>;
  Smem m;
  m.sA = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                    ~static_cast<uintptr_t>(1023));
  m.sB = m.sA + C::kStages * C::kATileBytes;
  m.sSF = m.sB + C::kStages * C::kBTileBytes;             // kSfGroups slots of kSfSlotBytes
  m.ss = reinterpret_cast<SharedState*>(m.sSF + kSfGroups * kSfSlotBytes);
  return m;
}

// Barriers and TMEM; warps 0 and 1.  The caller synchronises the CTA (and the cluster)
// before any role starts.
template <int kCta, bool kBlockScaled, int kTm = kBM>
__device__ __forceinline__ void gemm_init(const Smem& sm, const CUtensorMap* tmaps, int ntmaps) {
  SharedState& ss = *sm.ss;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < Cfg<kCta, kTm>::kStages; ++s) {
      mbar_init(&ss.full[s], 1);
      mbar_init(&ss.empty[s], 1);
    }
    for (int s = 0; s < kSfGroups; ++s) {
      mbar_init(&ss.sf_raw[s], 32);  // one cp.async completion arrival per loader lane
      mbar_init(&ss.sf_full[s], kCta);
      mbar_init(&ss.sf_empty[s], 1);
    }
    mbar_init(&ss.acc_full, 1);
    mbar_init(&ss.acc_empty, kEpiWarps * kCta);
    mbar_init(&ss.drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&ss.amax_bar[q], 64);  // every lane of both halves
    ss.abort = 0;
    ss.ready = 0;
    fence_barrier_init();
    for (int i = 0; i < ntmaps; ++i) tma_prefetch_desc(tmaps + i);
  }
  if (warp == 1) {
    if constexpr (kCta == 2) {
      tmem_alloc_pair(&ss.tmem_base, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&ss.tmem_base, kTmemCols);
      tmem_relinquish();
    }
  }
}

// m-block list of the expert offsets (warp 3; the caller synchronises after).  Every GEMM
// over the same offsets and tile shape shares it (tile t = m-block t / n_tiles, n-block
// t % n_tiles).
template <int kCta, int kTm = kBM>
__device__ __forceinline__ void gemm_prefix(const Smem& sm, const int32_t* offsets, int E) {
  using C = Cfg<kCta, kTm>;
  SharedState& ss = *sm.ss;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp != 3) return;
  int carry = 0;
  for (int base = 0; base <= E; base += 32) {
    const int e = base + lane;
    int o = 0, cnt = 0;
    if (e <= E) {
      o = __ldcg(offsets + e);
      ss.offs[e] = o;
    }
    if (e < E) cnt = (__ldcg(offsets + e + 1) - o + C::kTileM - 1) / C::kTileM;
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (e <= E) ss.mb_start[e] = carry + incl - cnt;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  __syncwarp();
  if (lane == 0) ss.mb_total = ss.mb_start[E];
}

// Releases TMEM (warp 1); the caller synchronises the CTA (and the cluster) first.
template <int kCta>
__device__ __forceinline__ void gemm_fini(const Smem& sm) {
  if ((threadIdx.x >> 5) == 1) {
    __syncwarp();
    if constexpr (kCta == 2) tmem_dealloc_pair(sm.ss->tmem_base, kTmemCols);
    else tmem_dealloc(sm.ss->tmem_base, kTmemCols);
  }
}

// One grouped GEMM over the tile list in shared memory (gemm_prefix), all roles.
// kCta: 1 (single) or 2 (pair).  kBlockScaled: false -> BF16 kind::f16; true ->
// kind::mxf8f6f4 with A = E4M3 and B = E4M3 (kBFmt 0) or E2M1 (kBFmt 5).  kSwiGLU: linear-1
// epilogue, else linear-2.  kOutE4M3: linear-1 stores h as E4M3 + 1x128 scales (else BF16).
// kStager: the MMA issuer polls the stager warp's ready count instead of waiting on the
// stage barriers itself (E2M1 weights only; gemm_phase picks it).  kDGate (with kSwiGLU,
// BF16): the backward form of linear-1, whose epilogue turns the recomputed pre-activations
// (g, u) and the gradient of h into the gradient of both (dg, du) instead of storing h.
template <int kCta, bool kBlockScaled, int kBFmt, bool kSwiGLU, bool kOutE4M3, int kTm,
          bool kStager, bool kDGate = false>
__device__ __forceinline__ void gemm_phase_k(const CUtensorMap* tmA_, const CUtensorMap* tmB_,
                                             const TcParams& p, const Smem& sm, Pipe& pipe) {
  using C = Cfg<kCta, kTm>;
  constexpr bool kPair = kCta == 2;
  constexpr int kStages = C::kStages;
  const CUtensorMap& tmA = *tmA_;
  const CUtensorMap& tmB = *tmB_;
  uint8_t* sA = sm.sA;
  uint8_t* sB = sm.sB;
  uint8_t* sSF = sm.sSF;
  SharedState& ss = *sm.ss;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const int cid = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int ncl = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  constexpr int kElemsPerRow = kBlockScaled ? 128 : 64;  // K elements per stage
  const int KB = p.K / kElemsPerRow;
  static_assert(!kStager || kBlockScaled, "the stager converts block scales");
  // tile order (every role decodes the same list): n-block-major inside an expert, so that
  // side-by-side CTAs share a weight tile, where a k-step's weight tile is the larger operand
  // (E4M3, BF16: 256 rows x 128 bytes against 128 x 128); for E2M1 weights the two are equal
  // and m-block-major, where they share the activation tile, measured faster
  constexpr bool kMbMajor = kBlockScaled && kBFmt == 5;
  const uint32_t tmem = ss.tmem_base;
  const int total = ss.mb_total * p.n_tiles;
  volatile int* abort = &ss.abort;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      constexpr uint32_t kBBytes = kBFmt == 5 ? C::kBTileBytes / 2 : C::kBTileBytes;
      constexpr uint32_t kCtaBytes = C::kATileBytes + kBBytes;
      uint32_t it = pipe.prod_it;
      const uint32_t it0 = it;
      for (int t = cid; t < total && !*abort; t += ncl) {
        const Tile tile = decode_tile(ss, p.E, p.n_tiles, C::kTileM, t, kMbMajor);
        const int arow = tile.m0 + static_cast<int>(rank) * kTm;
        // B rows of this CTA: linear-1 gate rows [nb*128, +128) then up rows [I + nb*128, +128);
        // linear-2 rows [nb*256, +256); a pair splits them between its two CTAs
        const int ebase = tile.e * p.w_rows;
        const int g0 = kSwiGLU ? ebase + tile.nb * 128 : ebase + tile.nb * kBN;
        const int g1 = kSwiGLU ? ebase + p.I + tile.nb * 128 : g0 + 128;
        const int brow = rank == 0 ? g0 : g1;
        for (int kb = 0; kb < KB; ++kb) {
          const int stage = static_cast<int>(it % kStages);
          const uint32_t phase = (it / kStages) & 1u;
          if (!mbar_wait<kPair>(&ss.empty[stage], phase ^ 1u, p.err, SITE_GEMM_EMPTY, abort)) break;
          const int kx = kb * kElemsPerRow;
          if constexpr (kPair) {
            if (rank == 0) mbar_arrive_expect_tx(&ss.full[stage], 2 * kCtaBytes);
            const uint32_t bar = mapa_shared(smem_u32(&ss.full[stage]), 0);
            tma_load_2d_pair(sA + stage * C::kATileBytes, &tmA, bar, kx, arow);
            tma_load_2d_pair(sB + stage * C::kBTileBytes, &tmB, bar, kx, brow);
          } else {
            mbar_arrive_expect_tx(&ss.full[stage], kCtaBytes);
            tma_load_2d(sA + stage * C::kATileBytes, &tmA, &ss.full[stage], kx, arow);
            tma_load_2d(sB + stage * C::kBTileBytes, &tmB, &ss.full[stage], kx, g0);
            tma_load_2d(sB + stage * C::kBTileBytes + C::kBTileBytes / 2, &tmB, &ss.full[stage], kx,
                        g1);
          }
          ++it;
        }
      }
      pipe.prod_it = it;
      if (*abort && rank == 0) {
        // drain: wait (bounded) for the copies of the last stages issued into this ring
        const uint32_t issued = it - it0;
        const uint32_t n = issued < static_cast<uint32_t>(kStages) ? issued : kStages;
        for (uint32_t i = 1; i <= n; ++i) {
          const int stage = static_cast<int>((it - i) % kStages);
          const uint32_t phase = ((it - i) / kStages) & 1u;
          const long long t0 = clock64();
          const long long limit = wait_limit(p.err);
          while (!mbar_try_wait_scoped<kPair>(&ss.full[stage], phase)) {
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
    if (lane == 0 && rank == 0) {
      constexpr int kMmaM = kBM * kCta;
      constexpr uint32_t kIdesc = kBlockScaled ? idesc_mxf8f6f4(kMmaM, kBN, 0u, kBFmt)
                                               : idesc_bf16(kMmaM, kBN);
      uint32_t it = pipe.mma_it, tiles = pipe.tiles, grp = pipe.sf_grp;
      uint32_t seen = 0;  // the stager's ready count as last observed
      bool issued_any = false;
      for (int t = cid; t < total && !*abort; t += ncl) {
        const uint32_t acc_phase = tiles & 1u;
        if (!mbar_wait<kPair>(&ss.acc_empty, acc_phase ^ 1u, p.err, SITE_GEMM_ACC_EMPTY, abort))
          break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          const int stage = static_cast<int>(it % kStages);
          // with the stager: it has seen this k-step's stage land (and converted its
          // scales); a shared-memory poll here instead of an mbarrier wait, which costs the
          // issuing thread far more than the MMAs' own issue
          if constexpr (kStager) {
            if (seen < it + 1u) {
              seen = wait_ready(&ss.ready, it + 1u, p.err, abort);
              if (seen == 0) {
                ok = false;
                break;
              }
            }
          } else {
            if (!mbar_wait<kPair>(&ss.full[stage], (it / kStages) & 1u, p.err, SITE_GEMM_FULL,
                                  abort)) {
              ok = false;
              break;
            }
          }
          const bool grp_start = (kb & 3) == 0;
          const bool grp_end = (kb & 3) == 3 || kb == KB - 1;
          // this k-step's group: grp counts the groups started so far (this one included
          // once its first k-step has passed)
          const uint32_t gcur = grp_start ? grp : grp - 1u;
          const int slot = static_cast<int>(gcur % kSfGroups);
          if constexpr (kBlockScaled && !kStager) {
            if (grp_start) {
              if (!mbar_wait<kPair>(&ss.sf_full[slot], (gcur / kSfGroups) & 1u, p.err,
                                    SITE_GEMM_FULL, abort)) {
                ok = false;
                break;
              }
            }
          }
          tc_fence_after();
          const uint64_t adesc = desc_kmajor_sw128(smem_u32(sA + stage * C::kATileBytes));
          const uint64_t bdesc = desc_kmajor_sw128(smem_u32(sB + stage * C::kBTileBytes));
          if (grp_start) ++grp;
          // A scales (and E4M3 B scales) are per 128 of K, so one byte per k-step: a group of
          // 4 k-steps shares one copy, byte kb % 4 selecting the k-step.  E2M1 B scales are per
          // 32 of K (byte = sub-block) and are copied every k-step.
          const uint32_t tsfa = tmem + kSfaCol + (grp % kSfSets) * kSfSetCols;
          const uint32_t tsfb =
              tmem + kSfbCol + (kBFmt == 5 ? it % kSfSets : grp % kSfSets) * kSfSetCols;
          if constexpr (kBlockScaled) {
            const uint32_t sf = smem_u32(sSF + slot * kSfSlotBytes);
            if (grp_start) {
              if constexpr (kPair) tc_cp_32x128b_warpx4_pair(tsfa, desc_sf_32x16(sf));
              else tc_cp_32x128b_warpx4(tsfa, desc_sf_32x16(sf));
            }
            if (kBFmt == 5 || grp_start) {
              // E2M1: this k-step's 2 atoms; E4M3: the group's 2 atoms
              const uint32_t sfb = sf + kSfBOff + (kBFmt == 5 ? 1024u * static_cast<uint32_t>(kb & 3) : 0u);
              if constexpr (kPair) {
                tc_cp_32x128b_warpx4_pair(tsfb, desc_sf_32x16(sfb));
                tc_cp_32x128b_warpx4_pair(tsfb + 4, desc_sf_32x16(sfb + 512));
              } else {
                tc_cp_32x128b_warpx4(tsfb, desc_sf_32x16(sfb));
                tc_cp_32x128b_warpx4(tsfb + 4, desc_sf_32x16(sfb + 512));
              }
            }
          }
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            // advance 32 bytes of K inside the 128-byte swizzle atom
            const uint64_t ad = adesc + static_cast<uint64_t>(ks * 2);
            const uint64_t bd = bdesc + static_cast<uint64_t>(ks * 2);
            const uint32_t acc = (kb | ks) != 0 ? 1u : 0u;
            if constexpr (kBlockScaled) {
              const uint32_t a_id = static_cast<uint32_t>(kb & 3);
              const uint32_t b_id = kBFmt == 5 ? static_cast<uint32_t>(ks) : a_id;
              const uint32_t id = kIdesc | (b_id << 4) | (a_id << 29);
              const uint32_t sfa = tsfa | (a_id << 30);
              const uint32_t sfb = tsfb | (b_id << 30);
              if constexpr (kPair) mma_mxf8f6f4_pair(tmem + kAccCol, ad, bd, id, sfa, sfb, acc);
              else mma_mxf8f6f4(tmem + kAccCol, ad, bd, id, sfa, sfb, acc);
            } else {
              if constexpr (kPair) mma_bf16_pair(tmem + kAccCol, ad, bd, kIdesc, acc);
              else mma_bf16(tmem + kAccCol, ad, bd, kIdesc, acc);
            }
          }
          issued_any = true;
          if constexpr (kPair) tc_commit_pair(&ss.empty[stage], 0x3);
          else tc_commit(&ss.empty[stage]);
          if constexpr (kBlockScaled) {
            if (grp_end) {  // the group's slot is free once its last k-step's MMAs are done
              if constexpr (kPair) tc_commit_pair(&ss.sf_empty[slot], 0x3);
              else tc_commit(&ss.sf_empty[slot]);
            }
          }
          ++it;
        }
        if (!ok) break;
        if constexpr (kPair) tc_commit_pair(&ss.acc_full, 0x3);
        else tc_commit(&ss.acc_full);
        ++tiles;
      }
      pipe.mma_it = it;
      pipe.tiles = tiles;
      pipe.sf_grp = grp;
      if (*abort && issued_any) {
        // let the issued MMAs finish before TMEM is released
        if constexpr (kPair) tc_commit_pair(&ss.drain, 0x1);
        else tc_commit(&ss.drain);
        const long long t0 = clock64();
        const long long limit = wait_limit(p.err);
        while (!mbar_try_wait_scoped<kPair>(&ss.drain, 0)) {
          if (clock64() - t0 > limit) break;
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------------ scale loader
    // Groups g = (tile, 4 consecutive k-steps) of this CTA in order; group g uses scale slot
    // g % kSfGroups.  Each lane copies the raw scales of its rows straight into the slot with
    // asynchronous copies (one 16-byte copy per row and group where the rows are 16-byte
    // aligned and the group is whole, else one 4-byte copy per k-step) whose completion
    // arrives on the slot's raw barrier, so the loader runs up to kSfGroups groups ahead of
    // the MMA issuer with nothing held in registers; row pointers are set up once per tile.
    // Each CTA copies the scales of its own 128 A rows and those the tile's B rows need; the
    // converter warp then rewrites the slot in place.
    if constexpr (kBlockScaled) {
      constexpr int kNB = kBFmt == 5 ? 8 : 2;  // B rows (E2M1) or weight blocks (E4M3) per lane
      const int KS = p.K / 128;                // fp32 scale columns of A (and of E4M3 B)
      const int NG = (KB + 3) / 4;             // groups per tile
      // 16-byte copies need the base pointer and every row start 16-byte aligned
      const bool a16 = (KS % 4) == 0 && (reinterpret_cast<uintptr_t>(p.a_scales) & 15u) == 0;
      const bool b16 = (kBFmt == 5 ? ((p.K / 32) % 16) == 0 : (KS % 4) == 0) &&
                       (reinterpret_cast<uintptr_t>(p.b_scales) & 15u) == 0;
      const float* pa[4];
      const uint8_t* pb[kNB];
      const int my_tiles = total > cid ? (total - cid + ncl - 1) / ncl : 0;
      const uint32_t g0 = pipe.sf_it;
      uint32_t gi = g0;
      bool ok = true;
      for (int lt = cid; lt < total && ok; lt += ncl) {
        const Tile tile = decode_tile(ss, p.E, p.n_tiles, C::kTileM, lt, kMbMajor);
        // only the tile's own rows are staged: the MMA's other rows (past the expert's end,
        // or past a small tile's 32) are never stored, and their scales may not exist yet
        uint32_t arow_ok = 0;
#pragma unroll
        for (int r1 = 0; r1 < 4; ++r1) {
          const int m = tile.m0 + static_cast<int>(rank) * kBM + lane + 32 * r1;
          if (lane + 32 * r1 < kTm && m < tile.m_end) arow_ok |= 1u << r1;
          pa[r1] = p.a_scales + static_cast<size_t>(m < p.S ? m : p.S - 1) * KS;
        }
        const int wr0 = kSwiGLU ? tile.nb * 128 : tile.nb * kBN;     // first B row, atom 0
        const int wr1 = kSwiGLU ? p.I + tile.nb * 128 : wr0 + 128;   // first B row, atom 1
        if constexpr (kBFmt == 5) {
          // lane l stages rows 128a + 32c + l of the tile (a = atom, c = 0..3)
#pragma unroll
          for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              int wr = (a == 0 ? wr0 : wr1) + lane + 32 * c;
              wr = wr < p.w_rows ? wr : p.w_rows - 1;
              pb[a * 4 + c] = static_cast<const uint8_t*>(p.b_scales) +
                              (static_cast<size_t>(tile.e) * p.w_rows + wr) * (p.K / 32);
            }
        } else {
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            int wr = a == 0 ? wr0 : wr1;
            wr = wr < p.w_rows ? wr : p.w_rows - 1;
            pb[a] = reinterpret_cast<const uint8_t*>(
                static_cast<const float*>(p.b_scales) +
                (static_cast<size_t>(tile.e) * (p.w_rows / 128) + wr / 128) * KS);
          }
        }
        for (int g = 0; g < NG; ++g, ++gi) {
          const int slot = static_cast<int>(gi % kSfGroups);
          if (!mbar_wait<kPair>(&ss.sf_empty[slot], ((gi / kSfGroups) & 1u) ^ 1u, p.err,
                                SITE_GEMM_SF_EMPTY, abort)) {
            ok = false;
            break;
          }
          uint8_t* sf = sSF + slot * kSfSlotBytes;
          const int nk = min(4, KB - 4 * g);  // k-steps in this group
          const bool whole = nk == 4;
#pragma unroll
          for (int r1 = 0; r1 < 4; ++r1) {
            if (!(arow_ok & (1u << r1))) continue;
            uint8_t* dst = sf + 16 * (lane + 32 * r1);
            const float* src = pa[r1] + 4 * g;
            if (a16 && whole) {
              cp_async_16(dst, src);
            } else {
              for (int j = 0; j < nk; ++j) cp_async_4(dst + 4 * j, src + j);
            }
          }
          if constexpr (kBFmt == 5) {
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              uint8_t* dst = sf + kSfBOff + 16 * (128 * (r >> 2) + 32 * (r & 3) + lane);
              const uint8_t* src = pb[r] + 16 * g;
              if (b16 && whole) {
                cp_async_16(dst, src);
              } else {
                for (int j = 0; j < nk; ++j) cp_async_4(dst + 4 * j, src + 4 * j);
              }
            }
          } else if (lane < 2) {
            uint8_t* dst = sf + kSfBRawE4 + 16 * lane;
            const float* src = reinterpret_cast<const float*>(pb[lane]) + 4 * g;
            if (b16 && whole) {
              cp_async_16(dst, src);
            } else {
              for (int j = 0; j < nk; ++j) cp_async_4(dst + 4 * j, src + j);
            }
          }
          cp_async_mbar_arrive(&ss.sf_raw[slot]);
        }
      }
      cp_async_wait_all();  // no copy may still be landing when the CTA moves on
      pipe.sf_it = g0 + static_cast<uint32_t>(my_tiles * NG);
    }
  } else if (kStager && warp == 3) {
    // ------------------------------------------------------------------ stager
    // Walks this CTA's k-steps in the MMA issuer's order.  At a group's first k-step of a
    // block-scaled kind it rewrites the group's staged raw scales in place into the layout
    // tcgen05.cp reads: per 128-row atom, 32 lines of 16 bytes, line l word c for row
    // 32c + l, one UE8M0 per byte.  A and E4M3 B scales cover 128 of K, so byte j of a word
    // is k-step j of the group (one TMEM copy per group; the MMA's scale-byte selector picks
    // the k-step); the UE8M0 byte of a power-of-two fp32 scale is its exponent field.  E2M1 B
    // scales are per 32 of K and already UE8M0: each k-step gets its own 2 atoms (byte =
    // sub-block).  Lane l reads only rows congruent to l mod 32 and writes only lines that
    // held such rows, so the in-place rewrite needs no exchange between lanes.  Then it waits
    // for the k-step's A/B stage to land and publishes the count of ready k-steps, which the
    // MMA issuer polls: the mbarrier waits run here, off the issuing thread.  In a pair both
    // CTAs convert their own scales and the leader's stager waits for the peer's before
    // publishing.  A scale word that is not a positive normal power of two (no exact UE8M0
    // byte) is reported once at the end as MOE_ERR_UNSUPPORTED.
    uint32_t it = pipe.st_it;  // k-steps, the MMA issuer's sequence
    uint32_t gi = pipe.sf_it;  // groups, the scale loader's sequence
    const uint32_t full_lead0 = mapa_shared(smem_u32(&ss.sf_full[0]), 0);
    uint32_t bad = 0;  // a scale word that is not a positive normal power of two was seen
    bool ok = true;
    for (int lt = cid; lt < total && ok; lt += ncl) {
      uint32_t arow_ok = 0;  // rows of this tile this lane converts (as the loader staged them)
      if constexpr (kBlockScaled) {
        const Tile tile = decode_tile(ss, p.E, p.n_tiles, C::kTileM, lt, kMbMajor);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int m = tile.m0 + static_cast<int>(rank) * kBM + lane + 32 * c;
          if (lane + 32 * c < kTm && m < tile.m_end) arow_ok |= 1u << c;
        }
      }
      for (int kb = 0; kb < KB; ++kb, ++it) {
        if constexpr (kBlockScaled) {
          if ((kb & 3) == 0) {
            const int slot = static_cast<int>(gi % kSfGroups);
            if (!mbar_wait(&ss.sf_raw[slot], (gi / kSfGroups) & 1u, p.err, SITE_GEMM_SF_EMPTY,
                           abort)) {
              ok = false;
              break;
            }
            uint8_t* sf = sSF + slot * kSfSlotBytes;
            const int nk = min(4, KB - kb);
            // A: rows lane + 32c -> line lane
            uint32_t wa[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 v = *reinterpret_cast<const uint4*>(sf + 16 * (lane + 32 * c));
              const uint32_t x[4] = {v.x, v.y, v.z, v.w};
              uint32_t w = 0;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                if (j < nk) {
                  w |= ((x[j] >> 23) & 0xFFu) << (8 * j);
                  if (arow_ok & (1u << c)) bad |= not_pow2_scale(x[j]);
                }
              }
              wa[c] = w;
            }
            *reinterpret_cast<uint4*>(sf + 16 * lane) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
            if constexpr (kBFmt == 5) {
              // rows 128a + 32c + lane, 16 B each (k-step j = word j) -> line (k-step j, atom a)
              uint4 v[2][4];
#pragma unroll
              for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                  v[a][c] = *reinterpret_cast<const uint4*>(sf + kSfBOff + 16 * (128 * a + 32 * c + lane));
#pragma unroll
              for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                  const uint32_t w0 = j == 0 ? v[a][0].x : j == 1 ? v[a][0].y : j == 2 ? v[a][0].z : v[a][0].w;
                  const uint32_t w1 = j == 0 ? v[a][1].x : j == 1 ? v[a][1].y : j == 2 ? v[a][1].z : v[a][1].w;
                  const uint32_t w2 = j == 0 ? v[a][2].x : j == 1 ? v[a][2].y : j == 2 ? v[a][2].z : v[a][2].w;
                  const uint32_t w3 = j == 0 ? v[a][3].x : j == 1 ? v[a][3].y : j == 2 ? v[a][3].z : v[a][3].w;
                  *reinterpret_cast<uint4*>(sf + kSfBOff + 1024 * j + 512 * a + 16 * lane) =
                      make_uint4(w0, w1, w2, w3);
                }
            } else {
              // the two weight blocks' scales, the same for every row of their atom
              const uint4 rg = *reinterpret_cast<const uint4*>(sf + kSfBRawE4);
              const uint4 ru = *reinterpret_cast<const uint4*>(sf + kSfBRawE4 + 16);
              const uint32_t xg[4] = {rg.x, rg.y, rg.z, rg.w}, xu[4] = {ru.x, ru.y, ru.z, ru.w};
              uint32_t wb0 = 0, wb1 = 0;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                if (j < nk) {
                  wb0 |= ((xg[j] >> 23) & 0xFFu) << (8 * j);
                  wb1 |= ((xu[j] >> 23) & 0xFFu) << (8 * j);
                  bad |= not_pow2_scale(xg[j]) | not_pow2_scale(xu[j]);
                }
              }
              *reinterpret_cast<uint4*>(sf + kSfBOff + 16 * lane) = make_uint4(wb0, wb0, wb0, wb0);
              *reinterpret_cast<uint4*>(sf + kSfBOff + 512 + 16 * lane) =
                  make_uint4(wb1, wb1, wb1, wb1);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if constexpr (kPair) {
              if (lane == 0) mbar_arrive_cluster(full_lead0 + slot * sizeof(uint64_t));
              if (rank == 0 && !mbar_wait<true>(&ss.sf_full[slot], (gi / kSfGroups) & 1u, p.err,
                                                SITE_GEMM_FULL, abort)) {
                ok = false;
                break;
              }
            } else if (lane == 0) {
              // nobody waits on it here, but a later phase without the stager (a short K
              // loop in the persistent kernel) reads this slot's phase
              mbar_arrive(&ss.sf_full[slot]);
            }
            ++gi;
          }
        }
        if (rank == 0) {
          const int stage = static_cast<int>(it % kStages);
          if (!mbar_wait<kPair>(&ss.full[stage], (it / kStages) & 1u, p.err, SITE_GEMM_FULL,
                                abort)) {
            ok = false;
            break;
          }
          __syncwarp();
          if (lane == 0) st_release_shared(&ss.ready, it + 1u);
        }
      }
    }
    pipe.st_it = it;
    pipe.sf_it = gi;
    // the exponent fields were used all the same: the result is undefined, the call fails
    if (bad) report_error(p.err, MOE_ERR_UNSUPPORTED, SITE_SCALE_FORMAT);
  } else if (warp == 3) {
    // ------------------------------------------------------------------ scale converter
    // Rewrites each staged group in place into the layout tcgen05.cp reads: per 128-row
    // atom, 32 lines of 16 bytes, line l word c for row 32c + l, one UE8M0 per byte.  A and
    // E4M3 B scales cover 128 of K, so byte j of a word is k-step j of the group (one TMEM
    // copy per group; the MMA's scale-byte selector picks the k-step); the UE8M0 byte of a
    // power-of-two fp32 scale is its exponent field.  E2M1 B scales are per 32 of K and
    // already UE8M0: each k-step gets its own 2 atoms (byte = sub-block).  Lane l reads only
    // rows congruent to l mod 32 and writes only lines that held such rows, so the in-place
    // rewrite needs no exchange between lanes.  A scale word that is not a positive normal
    // power of two (no exact UE8M0 byte) is reported once at the end as MOE_ERR_UNSUPPORTED.
    if constexpr (kBlockScaled) {
      const int NG = (KB + 3) / 4;
      const int my_tiles = total > cid ? (total - cid + ncl - 1) / ncl : 0;
      const int n_grp = my_tiles * NG;
      const uint32_t g0 = pipe.sf_it;
      const uint32_t full_lead0 = mapa_shared(smem_u32(&ss.sf_full[0]), 0);
      uint32_t bad = 0;  // a scale word that is not a positive normal power of two was seen
      uint32_t arow_ok = 0;  // rows of the current tile this lane converts (as the loader)
      for (int i = 0; i < n_grp; ++i) {
        const uint32_t gi = g0 + static_cast<uint32_t>(i);
        const int slot = static_cast<int>(gi % kSfGroups);
        if (i % NG == 0) {
          const Tile tile =
              decode_tile(ss, p.E, p.n_tiles, C::kTileM, cid + (i / NG) * ncl, kMbMajor);
          arow_ok = 0;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int m = tile.m0 + static_cast<int>(rank) * kBM + lane + 32 * c;
            if (lane + 32 * c < kTm && m < tile.m_end) arow_ok |= 1u << c;
          }
        }
        if (!mbar_wait(&ss.sf_raw[slot], (gi / kSfGroups) & 1u, p.err, SITE_GEMM_SF_EMPTY, abort))
          break;
        uint8_t* sf = sSF + slot * kSfSlotBytes;
        const int nk = min(4, KB - 4 * (i % NG));
        // A: rows lane + 32c -> line lane
        uint32_t wa[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(sf + 16 * (lane + 32 * c));
          const uint32_t x[4] = {v.x, v.y, v.z, v.w};
          uint32_t w = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (j < nk) {
              w |= ((x[j] >> 23) & 0xFFu) << (8 * j);
              if (arow_ok & (1u << c)) bad |= not_pow2_scale(x[j]);
            }
          }
          wa[c] = w;
        }
        *reinterpret_cast<uint4*>(sf + 16 * lane) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
        if constexpr (kBFmt == 5) {
          // rows 128a + 32c + lane, 16 B each (k-step j = word j) -> line (k-step j, atom a)
          uint4 v[2][4];
#pragma unroll
          for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c)
              v[a][c] = *reinterpret_cast<const uint4*>(sf + kSfBOff + 16 * (128 * a + 32 * c + lane));
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int a = 0; a < 2; ++a) {
              const uint32_t w0 = j == 0 ? v[a][0].x : j == 1 ? v[a][0].y : j == 2 ? v[a][0].z : v[a][0].w;
              const uint32_t w1 = j == 0 ? v[a][1].x : j == 1 ? v[a][1].y : j == 2 ? v[a][1].z : v[a][1].w;
              const uint32_t w2 = j == 0 ? v[a][2].x : j == 1 ? v[a][2].y : j == 2 ? v[a][2].z : v[a][2].w;
              const uint32_t w3 = j == 0 ? v[a][3].x : j == 1 ? v[a][3].y : j == 2 ? v[a][3].z : v[a][3].w;
              *reinterpret_cast<uint4*>(sf + kSfBOff + 1024 * j + 512 * a + 16 * lane) =
                  make_uint4(w0, w1, w2, w3);
            }
        } else {
          // the two weight blocks' scales, the same for every row of their atom
          const uint4 rg = *reinterpret_cast<const uint4*>(sf + kSfBRawE4);
          const uint4 ru = *reinterpret_cast<const uint4*>(sf + kSfBRawE4 + 16);
          const uint32_t xg[4] = {rg.x, rg.y, rg.z, rg.w}, xu[4] = {ru.x, ru.y, ru.z, ru.w};
          uint32_t wb0 = 0, wb1 = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (j < nk) {
              wb0 |= ((xg[j] >> 23) & 0xFFu) << (8 * j);
              wb1 |= ((xu[j] >> 23) & 0xFFu) << (8 * j);
              bad |= not_pow2_scale(xg[j]) | not_pow2_scale(xu[j]);
            }
          }
          *reinterpret_cast<uint4*>(sf + kSfBOff + 16 * lane) = make_uint4(wb0, wb0, wb0, wb0);
          *reinterpret_cast<uint4*>(sf + kSfBOff + 512 + 16 * lane) = make_uint4(wb1, wb1, wb1, wb1);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if constexpr (kPair) mbar_arrive_cluster(full_lead0 + slot * sizeof(uint64_t));
          else mbar_arrive(&ss.sf_full[slot]);
        }
      }
      pipe.sf_it = g0 + static_cast<uint32_t>(n_grp);
      // the k-steps the MMA issuer consumed in this phase: a later phase with the stager
      // publishes ready counts in the issuer's own sequence
      pipe.st_it += static_cast<uint32_t>(my_tiles * KB);
      // the exponent fields were used all the same: the result is undefined, the call fails
      if (bad) report_error(p.err, MOE_ERR_UNSUPPORTED, SITE_SCALE_FORMAT);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;             // TMEM lane quadrant (the warp's 32 rows)
    const int half = (warp - 4) >> 2;   // column half of the accumulator this warp reads
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t tiles = pipe.tiles, hq = pipe.hq;
    const uint32_t acc_empty_lead = mapa_shared(smem_u32(&ss.acc_empty), 0);
    for (int t = cid; t < total && !*abort; t += ncl) {
      const uint32_t acc_phase = tiles & 1u;
      const Tile tile = decode_tile(ss, p.E, p.n_tiles, C::kTileM, t, kMbMajor);
      // every lane waits; the decision is made warp-uniform so that the .sync.aligned
      // TMEM loads below always run with the full warp
      const bool ready =
          mbar_wait<kPair>(&ss.acc_full, acc_phase, p.err, SITE_GEMM_ACC_FULL, abort);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const int row0 = tile.m0 + static_cast<int>(rank) * kTm + q * 32;  // the warp's first row
      const int row = row0 + lane;
      const bool valid = q * 32 + lane < kTm && row < tile.m_end;
      // rows of this warp that exist (the tile's rows of this CTA, up to the expert's end)
      const int rows_ok = min(kTm - q * 32, tile.m_end - row0);
      // the warp's 128 accumulator columns: linear-1 gate [64h, 64h+64) and up
      // [128 + 64h, +64); linear-2 [128h, 128h + 128)
      uint32_t d[128];
      if constexpr (kSwiGLU) {
        tmem_ld32(trow + kAccCol + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(d));
        tmem_ld32(trow + kAccCol + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(d + 32));
        tmem_ld32(trow + kAccCol + 128 + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(d + 64));
        tmem_ld32(trow + kAccCol + 160 + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(d + 96));
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(trow + kAccCol + 128 * half + 32 * c,
                    *reinterpret_cast<uint32_t(*)[32]>(d + 32 * c));
      }
      tmem_ld_wait();
      // the accumulator is in registers: hand TMEM back before any arithmetic
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kPair) mbar_arrive_cluster(acc_empty_lead);
        else mbar_arrive(&ss.acc_empty);
      }
      if constexpr (kSwiGLU && kDGate) {
        // h = silu(g) u: dg = dh u silu'(g) = dh u s (1 + g (1 - s)), du = dh silu(g) = dh g s
        // with s = sigmoid(g), on the fp32 accumulator; the row's 64 columns of dh come in
        // (16-byte loads), its 64 gate and 64 up columns of dG [S, 2I] go out
        if (valid) {
          const int col0 = tile.nb * 128 + 64 * half;
          const uint4* dhp = reinterpret_cast<const uint4*>(
              static_cast<const __nv_bfloat16*>(p.dh) + static_cast<size_t>(row) * p.n_out + col0);
          __nv_bfloat16* dg_row = static_cast<__nv_bfloat16*>(p.out) +
                                  static_cast<size_t>(row) * 2 * p.n_out + col0;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 dv = __ldg(dhp + v);
            const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
            uint32_t wg[4], wu[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 dd = __bfloat1622float2(d2[i]);
              float rg[2], ru[2];
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                const float g = __uint_as_float(d[8 * v + 2 * i + c]);
                const float u = __uint_as_float(d[64 + 8 * v + 2 * i + c]);
                const float dhv = c == 0 ? dd.x : dd.y;
                const float sg = 1.0f / (1.0f + expf(-g));
                rg[c] = dhv * u * sg * (1.0f + g * (1.0f - sg));
                ru[c] = dhv * g * sg;
              }
              const __nv_bfloat162 bg = __floats2bfloat162_rn(rg[0], rg[1]);
              const __nv_bfloat162 bu = __floats2bfloat162_rn(ru[0], ru[1]);
              wg[i] = *reinterpret_cast<const uint32_t*>(&bg);
              wu[i] = *reinterpret_cast<const uint32_t*>(&bu);
            }
            reinterpret_cast<uint4*>(dg_row)[v] = make_uint4(wg[0], wg[1], wg[2], wg[3]);
            reinterpret_cast<uint4*>(dg_row + p.n_out)[v] = make_uint4(wu[0], wu[1], wu[2], wu[3]);
          }
        }
      } else if constexpr (kSwiGLU) {
        float h[64];
#pragma unroll
        for (int i = 0; i < 64; ++i)
          h[i] = silu_mul(__uint_as_float(d[i]), __uint_as_float(d[64 + i]));
        if constexpr (kOutE4M3) {
          // one power-of-two scale per 128 h columns = the whole tile row: the two halves
          // of the row exchange their partial amax
          // of the row exchange the scale exponent of their partial amax: the exponent rule
          // is monotonic in amax, so the row's exponent is the larger of the two (an
          // all-zero half contributes nothing; an all-zero row takes scale 1)
          float amax = 0.0f;
#pragma unroll
          for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(h[i]));
          constexpr int kNoExp = -128;
          const int own = amax > 0.0f ? max(e4m3_scale_exponent(amax), -126) : kNoExp;
          const int slot = static_cast<int>(hq & 1u);
          ss.ecode[slot][half][q * 32 + lane] = static_cast<int8_t>(own);
          mbar_arrive(&ss.amax_bar[q]);
          const bool got = mbar_wait(&ss.amax_bar[q], hq & 1u, p.err, SITE_GEMM_AMAX, abort);
          ++hq;
          if (!__all_sync(0xffffffffu, got)) break;
          const int both = max(own, static_cast<int>(ss.ecode[slot][half ^ 1][q * 32 + lane]));
          const int e = both == kNoExp ? 0 : both;
          const float inv = exp2i(-e);
          if (valid) {
            uint8_t* dst = static_cast<uint8_t*>(p.out) + static_cast<size_t>(row) * p.n_out +
                           tile.nb * 128 + 64 * half;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int b = 16 * v + 4 * i;
                const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                    make_float2(h[b] * inv, h[b + 1] * inv), __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                    make_float2(h[b + 2] * inv, h[b + 3] * inv), __NV_SATFINITE, __NV_E4M3);
                w[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
              }
              reinterpret_cast<uint4*>(dst)[v] = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (half == 0) p.out_scales[static_cast<size_t>(row) * (p.n_out / 128) + tile.nb] = exp2i(e);
          }
        } else {
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                  static_cast<size_t>(row) * p.n_out +
                                                  tile.nb * 128 + 64 * half);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(h[8 * v + 2 * i], h[8 * v + 2 * i + 1]);
                w[i] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      } else {
        // pack the warp's 128 columns of the row to BF16: chunk k = words 4k..4k+3 =
        // columns nb*256 + 128*half + 8k .. + 8
        uint32_t w[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const __nv_bfloat162 b2 =
              __floats2bfloat162_rn(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1]));
          w[i] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        const int chunks_ok = min(16, (p.n_out - tile.nb * kBN - 128 * half) / 8);
        store_rows_coalesced<16>(
            w, reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(p.out) +
                                          static_cast<size_t>(row0) * p.n_out + tile.nb * kBN +
                                          128 * half),
            static_cast<size_t>(p.n_out) * 2, rows_ok, chunks_ok, lane);
      }
      ++tiles;
    }
    pipe.hq = hq;
    pipe.tiles = tiles;
  }

}

// One grouped GEMM phase.  E2M1 weights need two scale copies every k-step on the MMA-issuing
// thread; over a K loop of 8 or more k-steps the stager warp taking the stage-barrier waits
// off that thread is measured faster.  E4M3 and BF16 kinds issue far fewer copies, and
// shorter K loops do not amortise the hand-off: both lose more to it than they gain.  The
// choice is per phase; the pipeline counters stay in step across phases of either kind.
template <int kCta, bool kBlockScaled, int kBFmt, bool kSwiGLU, bool kOutE4M3, int kTm = kBM,
          bool kDGate = false>
__device__ __forceinline__ void gemm_phase(const CUtensorMap* tmA_, const CUtensorMap* tmB_,
                                           const TcParams& p, const Smem& sm, Pipe& pipe) {
  static_assert(!kDGate || (kSwiGLU && !kBlockScaled), "the backward form: BF16 linear-1");
  if constexpr (kBlockScaled && kBFmt == 5) {
    if (p.K >= 8 * 128) {
      gemm_phase_k<kCta, kBlockScaled, kBFmt, kSwiGLU, kOutE4M3, kTm, true, kDGate>(
          tmA_, tmB_, p, sm, pipe);
      return;
    }
  }
  gemm_phase_k<kCta, kBlockScaled, kBFmt, kSwiGLU, kOutE4M3, kTm, false, kDGate>(
      tmA_, tmB_, p, sm, pipe);
}

}  // namespace gemm
}  // namespace moe
