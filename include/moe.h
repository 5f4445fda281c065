/*
 * moe.h -- C ABI of libmoe.so, a B200 (sm_100a) fused MoE expert layer.
 *
 * The layer is the one the source pages describe: a router picks k experts per token,
 * tokens are dispatched to their experts, each expert applies linear-1 (gate and up
 * projections), SwiGLU and linear-2, and the expert outputs are combined with the gate
 * weights (jiqizhixin, "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了", section
 * "Mega MoE 是什么？", the paragraph on the conventional dispatch -> linear -> SwiGLU ->
 * linear -> combine pipeline and the paragraph on fusing it into one mega-kernel).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library allocates no
 *     memory.  Row-major, contiguous, 16-byte aligned (E2M1 weights: 32-byte aligned).
 *   - Work is enqueued asynchronously on `stream`; a call returns once its launches are
 *     enqueued.  Argument errors are returned synchronously, before anything is launched.
 *   - A failed launch returns MOE_ERR_CUDA.  A device-side failure (a bounded wait that
 *     gave up) is recorded in a per-device error word read by moe_get_device_error().
 *   - Shapes: T tokens, H hidden, E experts, k experts per token, I expert intermediate
 *     size, S = T*k dispatch slots.  Preconditions: T >= 1, 1 <= k <= min(E, 32),
 *     E <= 1024, H % 128 == 0, I % 128 == 0, S <= 2^31 - 1 (slot indices are 32-bit; a
 *     larger S returns MOE_ERR_UNSUPPORTED and sizes its workspace to 0).
 *   - Tensor formats (moe_dtype):
 *       MOE_F32   IEEE binary32
 *       MOE_BF16  bfloat16
 *       MOE_E4M3  OCP FP8 E4M3 codes, one byte each; activations carry one fp32
 *                 power-of-two scale per 1x128 block along the row, weights one fp32
 *                 power-of-two scale per 128x128 block
 *       MOE_E2M1  OCP MX FP4 codes, two per byte (element 2i in the low nibble), weights
 *                 only, one UE8M0 scale byte (value 2^(b-127)) per 1x32 block along K
 *     An fp32 scale must be a positive normal power of two (2^-126 .. 2^127): the tensor
 *     cores take it as a UE8M0 exponent byte.  A GEMM that reads any other scale value
 *     records MOE_ERR_UNSUPPORTED with site 301 in the device error word and its output
 *     is undefined (scale values live on the device, so this cannot be checked before the
 *     launch).
 *   - Supported (activation, weight) pairs: (F32, F32), (BF16, BF16), (E4M3, E4M3),
 *     (E4M3, E2M1).  h (the SwiGLU output) is stored in the activation format (E4M3 with a
 *     power-of-two scale per 1x128 block); y and out are BF16, except F32 for the F32 layer.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1, /* null pointer, bad shape or bad enum value */
  MOE_ERR_UNSUPPORTED = -2, /* valid but unsupported combination (dtype pair, E > 1024 ...) */
  MOE_ERR_MISALIGNED = -3,  /* a pointer misses its alignment requirement */
  MOE_ERR_WORKSPACE = -4,   /* workspace null, too small or not 256-byte aligned */
  MOE_ERR_CUDA = -5,        /* a CUDA runtime / driver call or a launch failed */
  MOE_ERR_TIMEOUT = -6,     /* device side: a bounded wait gave up (see moe_get_device_error) */
  MOE_ERR_DEVICE = -7       /* device side: any other recorded failure */
} moe_status;

typedef enum moe_dtype { MOE_F32 = 0, MOE_BF16 = 1, MOE_E4M3 = 2, MOE_E2M1 = 3 } moe_dtype;

typedef enum moe_score { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score;

/* Workspace queries name the entry point they size. */
typedef enum moe_op {
  MOE_OP_DISPATCH = 1,
  MOE_OP_LINEAR1 = 2,
  MOE_OP_LINEAR2 = 3,
  MOE_OP_FUSED_FFN = 4,
  MOE_OP_FORWARD = 5,
  MOE_OP_BACKWARD = 6
} moe_op;

/* Expert weights.  W1 [E, 2I, H]: rows [0, I) are the gate projection, rows [I, 2I) the up
 * projection.  W2 [E, H, I].  Both K-major (each output row contiguous over the reduction
 * dimension).  Scales: E4M3 -> fp32 [E, 2I/128, H/128] and [E, H/128, I/128];
 * E2M1 -> UE8M0 bytes [E, 2I, H/32] and [E, H, I/32]; F32 / BF16 -> NULL. */
/* What the fp32 block scales of an E4M3 layer hold (activation scales x_scales /
 * x_perm_scales and the E4M3 weight scales alike).
 *   MOE_SCALE_POW2  positive normal powers of two: they convert exactly to the UE8M0 scales
 *                   the block-scaled tensor-core MMA applies (the fast path; any other value
 *                   is reported on the device as MOE_ERR_UNSUPPORTED at site 301)
 *   MOE_SCALE_FP32  any positive finite fp32 values: the expert GEMMs run unscaled E4M3
 *                   MMAs per 128-deep block of K and fold each block's partial sum into an
 *                   fp32 accumulator with its scales (E4M3 weights only; the layer runs as
 *                   the chain of entry points, also under moe_forward) */
typedef enum moe_scale_fmt { MOE_SCALE_POW2 = 0, MOE_SCALE_FP32 = 1 } moe_scale_fmt;

typedef struct moe_weights {
  int act; /* moe_dtype of x, x_perm and h */
  int wt;  /* moe_dtype of W1 and W2 */
  const void* w1;
  const void* w1_scales;
  const void* w2;
  const void* w2_scales;
  int scale_fmt; /* moe_scale_fmt (0, the power-of-two scales, when zero-initialised) */
} moe_weights;

/* Router: per token, select k experts and their gate weights.
 * (youleyou, "DeepSeek 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", section
 *  "Tile Kernels：逼近硬件极限的底层优化", gating item: top-k expert selection with scoring;
 *  routing item: weight normalisation.)
 *   logits   fp32 [T, E], finite (not checked on the device)
 *   bias     fp32 [E] or NULL; only MOE_SCORE_SIGMOID uses it, for selection only
 *   score    MOE_SCORE_SOFTMAX: select on the logits; gates = softmax over the selected k
 *                               (renorm) or the full softmax of the selected (no renorm).
 *            MOE_SCORE_SIGMOID: s = sigmoid(logit) evaluated as a fixed sequence of
 *                               correctly rounded fp32 operations; select on s + bias;
 *                               gates = s / sum(selected s) (renorm) or s.
 *   topk_idx int32 [T, k] out, experts in rank order (key descending, ties -> lower id)
 *   topk_w   fp32 [T, k] out, the gates in the same order */
moe_status moe_route(const float* logits, const float* bias, int T, int E, int k, int score,
                     int renorm, int32_t* topk_idx, float* topk_w, cudaStream_t stream);

/* Group-limited routing and the routed scaling factor, for moe_route_ex / moe_forward_ex.
 * The experts form n_group consecutive groups of G = E / n_group (G a multiple of 32, or
 * n_group = 1).  A group's score is the fp32 sum of its two largest selection keys (as
 * moe_route forms them); the topk_group best groups (equal scores -> lower group) are kept
 * and the k experts are selected among theirs only, in the same rank order.  The gates are
 * then multiplied by `scale`.  {1, 1, 1.0f} is moe_route itself.  Not on the source pages,
 * which only name gating with top-k selection and weight normalisation; this is the
 * DeepSeek-V3-style variant of it.
 *   errors: MOE_ERR_INVALID_ARG for n_group < 1, topk_group outside [1, n_group],
 *           k > topk_group * G or a non-finite scale; MOE_ERR_UNSUPPORTED when E is not a
 *           multiple of n_group or G is not a multiple of 32 (n_group > 1). */
typedef struct {
  int n_group;
  int topk_group;
  float scale;
} moe_router_groups;

/* moe_route with group-limited selection and a routed scaling factor (groups may be NULL:
 * moe_route). */
moe_status moe_route_ex(const float* logits, const float* bias, int T, int E, int k, int score,
                        int renorm, const moe_router_groups* groups, int32_t* topk_idx,
                        float* topk_w, cudaStream_t stream);

/* Dispatch: permute token rows to experts (stable counting sort by expert).
 * (jiqizhixin, section "Mega MoE 是什么？", pipeline paragraph: tokens are dispatched to the
 *  experts; youleyou, routing item: token-to-expert mapping with fused expand.)
 *   x              [T, H] in format `act` (F32, BF16 or E4M3)
 *   x_scales       fp32 [T, H/128] for E4M3, else NULL
 *   topk_idx       int32 [T, k] from moe_route (each expert at most once per token)
 *   x_perm         [S, H] out: slot p holds the row of token perm_src[p] / k
 *   x_perm_scales  fp32 [S, H/128] out for E4M3, else NULL
 *   expert_offsets int32 [E+1] out: slots of expert e are [offsets[e], offsets[e+1]),
 *                  in ascending token order
 *   perm_src       int32 [S] out: slot -> t*k + j
 *   slot_of        int32 [S] out: t*k + j -> slot
 *   ws             workspace of moe_workspace_size(MOE_OP_DISPATCH, ...) bytes, 256-byte
 *                  aligned, contents need no initialisation */
moe_status moe_dispatch(const void* x, const float* x_scales, int act, int T, int H, int E, int k,
                        const int32_t* topk_idx, void* x_perm, float* x_perm_scales,
                        int32_t* expert_offsets, int32_t* perm_src, int32_t* slot_of, void* ws,
                        size_t ws_bytes, cudaStream_t stream);

/* Dispatch of BF16 rows into an E4M3 layer: moe_dispatch with the activation quantisation
 * fused into the row copy.  Each 1x128 block of a token row gets the scale 2^n, n the
 * smallest integer with amax <= 448 * 2^n (an all-zero block gets 2^0; n >= -126), and codes
 * round to nearest even, saturating — the rule of the h requantisation; the codes are a
 * function of the input bits alone.
 * (youleyou, "DeepSeek 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", Tile Kernels feature
 *  list, quantisation item: FP8 per-block quantisation; jiqizhixin, "DeepSeek悄悄更新：Mega
 *  MoE、FP4 Indexer来了", FP8 x FP4 paragraph: FP8 activations.)
 *   x              BF16 [T, H] (16-byte aligned)
 *   x_perm         E4M3 codes [S, H] out;  x_perm_scales fp32 [S, H/128] out
 *   other arguments, outputs, workspace and errors as moe_dispatch. */
moe_status moe_dispatch_quant(const void* x, int T, int H, int E, int k,
                              const int32_t* topk_idx, void* x_perm, float* x_perm_scales,
                              int32_t* expert_offsets, int32_t* perm_src, int32_t* slot_of,
                              void* ws, size_t ws_bytes, cudaStream_t stream);

/* Expert linear-1 + SwiGLU (+ requantisation): for every slot p of expert e,
 *   gate = x_perm[p] . W1[e, 0:I]^T, up = x_perm[p] . W1[e, I:2I]^T (fp32 accumulation),
 *   h[p] = silu(gate) * up stored in format W->act; for E4M3 each 1x128 block of h gets the
 *   scale 2^n with n the smallest integer such that amax <= 448 * 2^n, and codes are
 *   round-to-nearest-even, saturating.
 * (jiqizhixin, section "Mega MoE 是什么？", pipeline paragraph: linear layer then SwiGLU;
 *  FP8 x FP4 paragraph; youleyou, quantisation item: FP8/FP4 quantisation fused with SwiGLU.)
 *   h        [S, I] out;  h_scales fp32 [S, I/128] out for E4M3, else NULL
 *   ws       may be NULL (this entry needs no workspace) */
moe_status moe_expert_linear1(const void* x_perm, const float* x_perm_scales,
                              const int32_t* expert_offsets, int S, int H, int I, int E,
                              const moe_weights* W, void* h, float* h_scales, void* ws,
                              size_t ws_bytes, cudaStream_t stream);

/* Expert linear-2: y[p] = h[p] . W2[e]^T for every slot p of expert e, fp32 accumulation,
 * stored BF16 (F32 for the F32 layer), unweighted.
 * (jiqizhixin, section "Mega MoE 是什么？", pipeline paragraph: the second linear layer.)
 *   h [S, I] (+ h_scales fp32 [S, I/128] for E4M3);  y [S, H] out;  ws may be NULL. */
moe_status moe_expert_linear2(const void* h, const float* h_scales, const int32_t* expert_offsets,
                              int S, int H, int I, int E, const moe_weights* W, void* y, void* ws,
                              size_t ws_bytes, cudaStream_t stream);

/* The expert FFN of the dispatched rows: linear-1 + SwiGLU (+ h requantisation for E4M3)
 * followed by linear-2, y[p] = W2[e] . SwiGLU(W1[e] . x_perm[p]) for every slot p of
 * expert e, with h kept in the workspace (moe_workspace_size(MOE_OP_FUSED_FFN, ...) bytes,
 * 256-byte aligned).
 * (jiqizhixin, section "Mega MoE 是什么？", pipeline paragraph: a linear layer, the SwiGLU
 *  activation and a second linear layer between dispatch and combine; youleyou, section
 *  "Tile Kernels：逼近硬件极限的底层优化", feature list, quantisation item: FP8 quantisation
 *  fused with SwiGLU.)
 *   Arguments as moe_expert_linear1 / moe_expert_linear2; y [S, H] out.  Errors: those of
 *   the two calls, and MOE_ERR_WORKSPACE for a missing, misaligned or short workspace. */
moe_status moe_fused_ffn(const void* x_perm, const float* x_perm_scales,
                         const int32_t* expert_offsets, int S, int H, int I, int E,
                         const moe_weights* W, void* y, void* ws, size_t ws_bytes,
                         cudaStream_t stream);

/* Combine: out[t] = sum_{j<k} topk_w[t, j] * y[slot_of[t*k + j]], accumulated in fp32 in
 * rank order j, no atomics (the result is deterministic), stored in out_dt.
 * (jiqizhixin, section "Mega MoE 是什么？", pipeline paragraph: results are put back
 *  together; youleyou, routing item: fused reduce.)
 *   y [S, H] in y_dt (BF16 or F32);  out [T, H] in out_dt (BF16 or F32). */
moe_status moe_combine(const void* y, int y_dt, const int32_t* slot_of, const float* topk_w,
                       int T, int k, int H, void* out, int out_dt, cudaStream_t stream);

/* The whole layer: route -> dispatch -> linear-1 + SwiGLU -> linear-2 -> combine, all
 * intermediates in the workspace (moe_workspace_size(MOE_OP_FORWARD, ...) bytes).
 * (jiqizhixin, section "Mega MoE 是什么？", the mega-kernel paragraph.)
 * For the tensor-core formats (BF16, E4M3 activations with power-of-two block scales) this
 * is ONE persistent cooperative kernel launch (plus an 8-byte memset of its grid barrier)
 * running every step in phases, with the expert GEMMs' tile shape the chain would use (for
 * 256-row CTA-pair tiles it is a cluster launch of as many pairs as can be resident at
 * once); it produces the same bytes as the chain moe_route, moe_dispatch,
 * moe_expert_linear1, moe_expert_linear2, moe_combine.  The fp32 layer and weights marked
 * MOE_SCALE_FP32 run that chain.
 * topk_idx / topk_w / expert_offsets may be NULL; when given, the routing result and the
 * per-expert offsets are written there too.
 * x is in format W->act with x_scales for E4M3; for E4M3 layers x_scales may instead be NULL,
 * and then x is BF16 [T, H] that the dispatch quantises as moe_dispatch_quant does. */
moe_status moe_forward(const void* x, const float* x_scales, const float* logits,
                       const float* bias, int score, int renorm, int T, int H, int E, int k,
                       int I, const moe_weights* W, void* out, int32_t* topk_idx,
                       float* topk_w, int32_t* expert_offsets, void* ws, size_t ws_bytes,
                       cudaStream_t stream);

/* moe_forward routed as moe_route_ex does (groups may be NULL: moe_forward). */
moe_status moe_forward_ex(const void* x, const float* x_scales, const float* logits,
                          const float* bias, int score, int renorm,
                          const moe_router_groups* groups, int T, int H, int E, int k, int I,
                          const moe_weights* W, void* out, int32_t* topk_idx, float* topk_w,
                          int32_t* expert_offsets, void* ws, size_t ws_bytes,
                          cudaStream_t stream);

/* Batched transpose: dst[e] = src[e]^T for src [E, R, C] row-major, dst [E, C, R].
 * (youleyou, section "Tile Kernels：逼近硬件极限的底层优化", feature list, batched matrix
 *  transpose item.)  Makes the transposed weight copies the backward's GEMMs read
 * (W1^T [E, H, 2I], W2^T [E, I, H]).
 *   dtype  element size: MOE_F32 (4 bytes), MOE_BF16 (2), MOE_E4M3 (1); E2M1 (packed
 *          nibbles) returns MOE_ERR_UNSUPPORTED.
 *   src, dst device buffers of E*R*C elements; they must not overlap. */
moe_status moe_transpose_experts(const void* src, int dtype, int E, int R, int C, void* dst,
                                 cudaStream_t stream);

/* Inputs and outputs of moe_expert_backward (all device pointers; S = T*k). */
typedef struct moe_backward_args {
  int T, H, E, k, I;
  int score;        /* moe_score of the forward router */
  int renorm;       /* the forward's renorm flag */
  float scale;      /* the forward's routed scaling factor (1 for moe_forward) */
  const void* dout; /* BF16 [T, H]: gradient of the layer output */
  const float* logits;           /* fp32 [T, E], as given to the forward */
  const int32_t* topk_idx;       /* int32 [T, k], the forward's selection */
  const float* topk_w;           /* fp32 [T, k], the forward's gates */
  const int32_t* expert_offsets; /* int32 [E+1]  (moe_dispatch) */
  const int32_t* slot_of;        /* int32 [T*k]  (moe_dispatch) */
  const void* x_perm;            /* BF16 [S, H]  (moe_dispatch) */
  const void* h;                 /* BF16 [S, I]  (moe_expert_linear1) */
  const void* y;                 /* BF16 [S, H]  (moe_expert_linear2) */
  const void* w1;                /* BF16 [E, 2I, H] */
  const void* w2;                /* BF16 [E, H, I] (read through w2_t only) */
  const void* w1_t;              /* BF16 [E, H, 2I] = W1^T (moe_transpose_experts) */
  const void* w2_t;              /* BF16 [E, I, H]  = W2^T (moe_transpose_experts) */
  void* dx;                      /* out BF16 [T, H] */
  float* dw1;                    /* out fp32 [E, 2I, H]; experts no token picked get 0 */
  float* dw2;                    /* out fp32 [E, H, I] */
  float* dlogits;                /* out fp32 [T, E] */
} moe_backward_args;

/* Backward of the BF16 layer: the gradients of out = sum_j w[t, j] * W2_e SwiGLU(W1_e x_t)
 * with respect to x, W1, W2 and the router logits, the top-k selection held fixed (it is
 * piecewise constant; the sigmoid router's selection bias gets no gradient).
 * (youleyou, section "Tile Kernels：逼近硬件极限的底层优化", feature list, model-layer item:
 *  wrappers that make the kernels trainable layers.)
 * Steps, each stored where the comment says:
 *   combine backward:  dy_w[slot] = BF16(w * dout[t]);  dgate = dout[t] . y[slot] (fp32)
 *   router backward:   dlogits (fp32) through the gate function
 *   dh = BF16(dy_w W2)       (expert GEMM on W2^T)
 *   dG = BF16(SwiGLU backward of (g, u), dh): the expert GEMM of linear-1 recomputes the
 *        pre-activations (g, u) = x_perm W1^T in fp32 and its epilogue turns them and dh
 *        into dg = dh u s (1 + g (1 - s)) and du = dh g s, s = sigmoid(g); g and u are
 *        not stored
 *   dx_slot = BF16(dG W1)    (expert GEMM on W1^T);  dx[t] = BF16(sum of its k slots)
 *   dW1_e = dG_e^T x_e,  dW2_e = dy_w,e^T h_e  (fp32; tensor cores, on copies of the
 *                                               operands transposed so that each expert's
 *                                               slots form a zero-padded 64-column segment)
 * BF16 layers only (the arguments carry no formats).  BF16 tensors, dw1 and dw2 must be
 * 16-byte aligned, the other arrays 4-byte aligned.  Workspace:
 * moe_workspace_size(MOE_OP_BACKWARD, T, H, E, k, I, MOE_BF16, MOE_BF16) bytes, 256-byte
 * aligned.  Deterministic: no atomics; every sum runs in a fixed order. */
moe_status moe_expert_backward(const moe_backward_args* args, void* ws, size_t ws_bytes,
                               cudaStream_t stream);

/* moe_dispatch without a caller workspace, for callers that cannot allocate device memory
 * (a host with no device allocator of its own, a runtime that forbids allocations after
 * start-up, or a path that must not call cudaMalloc / cudaFree because they can synchronise
 * the device).  The source pages have no counterpart to this entry point; it exists for
 * those callers only.
 *   Arguments, outputs and results are those of moe_dispatch, minus ws / ws_bytes.
 *   Scratch comes from a 4 MiB buffer compiled into the library, held by every device that
 *   loads it until the process exits.  Shapes whose dispatch workspace exceeds it
 *   (moe_workspace_size(MOE_OP_DISPATCH, ...) > 4 MiB; e.g. T > 32736 at E = 1024) return
 *   MOE_ERR_WORKSPACE before anything is launched.
 *   Every call looks up the buffer's device address on the caller's current device (no
 *   address is cached).  The first call on a device also loads the library's module there;
 *   make that first call before any stream capture.
 *   All calls on a device share the buffer: nothing needs clearing between calls, but calls
 *   that may overlap on the GPU (other streams, other host threads) race and must be
 *   serialised by the caller. */
moe_status moe_dispatch_noalloc(const void* x, const float* x_scales, int act, int T, int H, int E,
                                int k, const int32_t* topk_idx, void* x_perm,
                                float* x_perm_scales, int32_t* expert_offsets, int32_t* perm_src,
                                int32_t* slot_of, cudaStream_t stream);

/* Bytes of workspace entry point `op` needs for these shapes (0 for an invalid query). */
size_t moe_workspace_size(int op, int T, int H, int E, int k, int I, int act, int wt);

/* Synchronises `stream`, then reads and clears the calling device's error word.
 * Returns MOE_OK, or the first recorded failure with *site (may be NULL) set to the code
 * location that recorded it, or MOE_ERR_CUDA if the synchronisation itself failed.
 * Recorded failures: MOE_ERR_TIMEOUT at a bounded wait (sites 101-106: GEMM pipeline
 * barriers; 201: the persistent kernel's grid barrier; 901: the self-test's mbarrier),
 * MOE_ERR_UNSUPPORTED at site 301 (an fp32 block scale that is not a positive normal power
 * of two).  The wait limit (moe_set_wait_limit) is kept. */
moe_status moe_get_device_error(cudaStream_t stream, int* site);

/* Limit of every bounded wait in the library's kernels (mbarrier waits of the GEMM
 * pipeline and its drains, the persistent kernel's grid barriers), in SM clock cycles, for
 * the calling thread's current device (call once per device; it holds for every later
 * launch on that device, from any host thread).  0 restores the default of 2e9 cycles
 * (about one second at the B200's boost clock; legitimate waits take microseconds).  A wait
 * that runs past the limit records MOE_ERR_TIMEOUT and its site in the device error word
 * and its kernel returns without finishing the work, leaving the context usable.
 * Synchronous (a 8-byte copy to the device).  Returns MOE_ERR_INVALID_ARG for cycles < 0,
 * MOE_ERR_CUDA if the copy fails. */
moe_status moe_set_wait_limit(long long cycles);

/* Self-test of the bounded waits (failure detection; the source pages have no counterpart).
 * Launches a kernel whose wait can never be satisfied, by construction:
 *   MOE_SELFTEST_MBARRIER      one CTA waits on an mbarrier that nothing arrives on;
 *                              records MOE_ERR_TIMEOUT at site 901
 *   MOE_SELFTEST_GRID_BARRIER  every CTA of a cooperative grid (one per SM) arrives at a
 *                              grid barrier expecting one arrival more than the grid has;
 *                              records MOE_ERR_TIMEOUT at site 201
 * The kernel returns once the wait limit has passed; read the result with
 * moe_get_device_error.  Nothing traps, faults or waits without a limit.  Returns
 * MOE_ERR_INVALID_ARG for another kind, MOE_ERR_CUDA if the launch fails. */
enum { MOE_SELFTEST_MBARRIER = 0, MOE_SELFTEST_GRID_BARRIER = 1 };
moe_status moe_selftest_wait(int kind, cudaStream_t stream);

/* Static string naming a status code. */
const char* moe_status_string(int status);

/* Number of this library's kernel launches made since it was loaded (host-side counter,
 * for accounting in benchmarks). */
uint64_t moe_launch_count(void);

/* Process-wide tile shape of the tensor-core expert GEMMs (a tuning and testing knob):
 * 0 automatic, 1 always single CTAs (128-row tiles), 2 always CTA pairs (256-row tiles on
 * cta_group::2; moe_forward's single launch uses single CTAs instead), 3 always small tiles
 * (32-row m-blocks, one CTA).  Automatic: small tiles when S <= 16 * E (decode-sized
 * batches), pairs for BF16 when S >= 128 * E, single CTAs otherwise.  Single and small tiles
 * give identical bits; pairs are identical up to fp32 accumulation order.  Returns
 * MOE_ERR_INVALID_ARG for any other value. */
moe_status moe_set_gemm_tiles(int mode);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
