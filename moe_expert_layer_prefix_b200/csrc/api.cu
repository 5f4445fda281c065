// C ABI of libmoe.so: argument checking, workspace carving and launch sequencing.
// Every computation happens in the kernels of the other translation units.
#include <atomic>
#include <cstddef>
#include <climits>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {

// Per-device control block: the error word {status, site} that kernels whose waits are
// bounded write, followed by the wait limit they read (SM clock cycles).
struct DevCtl {
  int status;
  int site;
  long long wait_limit;
};
static_assert(offsetof(DevCtl, wait_limit) == 8, "kernels read the limit at err + 2");
__device__ DevCtl g_error_word = {0, 0, kWaitLimitCycles};

namespace {
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_tile_mode{0};

constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices] = {};
std::mutex g_mu;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}
}  // namespace

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

int gemm_tile_mode() { return g_tile_mode.load(); }

int* device_error_word() {
  // looked up on every call (cheap): a cached address would go stale after a device reset
  // or in another context on the same device
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

moe_status check_dispatch_shapes(int T, int H, int E, int k) {
  if (T < 1 || H < 128 || E < 1 || k < 1) return MOE_ERR_INVALID_ARG;
  if (H % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (E > 1024 || k > 32 || k > E || static_cast<long long>(T) * k > INT32_MAX)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int num_sms() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sms[d] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0)
      n = 148;
    g_sms[d] = n;
  }
  return g_sms[d];
}

}  // namespace moe

using namespace moe;

namespace {

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline size_t round256(size_t b) { return (b + 255) / 256 * 256; }

inline size_t act_bytes(int act) { return act == MOE_F32 ? 4 : act == MOE_BF16 ? 2 : 1; }

inline bool valid_pair(int act, int wt) {
  return (act == MOE_F32 && wt == MOE_F32) || (act == MOE_BF16 && wt == MOE_BF16) ||
         (act == MOE_E4M3 && (wt == MOE_E4M3 || wt == MOE_E2M1));
}

inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Slot indices t*k + j are 32-bit on the device.
inline bool slots_fit(int T, int k) { return static_cast<long long>(T) * k <= INT32_MAX; }

moe_status check_shapes(int T, int H, int E, int k) { return check_dispatch_shapes(T, H, E, k); }

moe_status check_weights(const moe_weights* W, int need_act) {
  if (W == nullptr || W->w1 == nullptr || W->w2 == nullptr) return MOE_ERR_INVALID_ARG;
  if (W->act < MOE_F32 || W->act > MOE_E2M1 || W->wt < MOE_F32 || W->wt > MOE_E2M1)
    return MOE_ERR_INVALID_ARG;
  if (need_act >= 0 && W->act != need_act) return MOE_ERR_INVALID_ARG;
  if (!valid_pair(W->act, W->wt)) return MOE_ERR_UNSUPPORTED;
  if (W->scale_fmt != MOE_SCALE_POW2 && W->scale_fmt != MOE_SCALE_FP32) return MOE_ERR_INVALID_ARG;
  if (W->scale_fmt == MOE_SCALE_FP32 && (W->act != MOE_E4M3 || W->wt != MOE_E4M3))
    return MOE_ERR_UNSUPPORTED;
  const bool scaled = W->wt == MOE_E4M3 || W->wt == MOE_E2M1;
  if (scaled && (W->w1_scales == nullptr || W->w2_scales == nullptr)) return MOE_ERR_INVALID_ARG;
  const size_t a = W->wt == MOE_E2M1 ? 32 : 16;
  if (!aligned(W->w1, a) || !aligned(W->w2, a)) return MOE_ERR_MISALIGNED;
  if (scaled && (!aligned(W->w1_scales, 4) || !aligned(W->w2_scales, 4))) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

size_t h_bytes(int S, int I, int act) {
  return round256(static_cast<size_t>(S) * I * act_bytes(act)) +
         (act == MOE_E4M3 ? round256(static_cast<size_t>(S) * (I / 128) * 4) : 0);
}

moe_status run_ffn(int which, const FfnArgs& a, cudaStream_t s) {
  cudaError_t e;
  if (a.act == MOE_F32) {
    e = which == 1 ? launch_linear1_simt(a, s) : launch_linear2_simt(a, s);
  } else {
    e = which == 1 ? launch_linear1_tc(a, s) : launch_linear2_tc(a, s);
  }
  return cuda_status(e);
}

}  // namespace

extern "C" {

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_MISALIGNED: return "MOE_ERR_MISALIGNED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
    default: return "MOE_ERR_UNKNOWN";
  }
}

uint64_t moe_launch_count(void) { return g_launches.load(); }

moe_status moe_set_wait_limit(long long cycles) {
  if (cycles < 0) return MOE_ERR_INVALID_ARG;
  const long long v = cycles == 0 ? kWaitLimitCycles : cycles;
  if (cudaMemcpyToSymbol(g_error_word, &v, sizeof(v), offsetof(DevCtl, wait_limit)) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_set_gemm_tiles(int mode) {
  if (mode < 0 || mode > 3) return MOE_ERR_INVALID_ARG;
  g_tile_mode.store(mode);
  return MOE_OK;
}

size_t moe_workspace_size(int op, int T, int H, int E, int k, int I, int act, int wt) {
  if (T < 1 || H < 1 || E < 1 || k < 1 || I < 1 || !slots_fit(T, k)) return 0;
  if (!valid_pair(act, wt)) return 0;
  const int S = T * k;
  switch (op) {
    case MOE_OP_DISPATCH:
      return dispatch_ws_bytes(T, E);
    case MOE_OP_LINEAR1:
    case MOE_OP_LINEAR2:
      return 0;
    case MOE_OP_FUSED_FFN:
      return h_bytes(S, I, act);
    case MOE_OP_BACKWARD: {
      if (act != MOE_BF16 || wt != MOE_BF16) return 0;
      size_t b = 0;
      b += round256(static_cast<size_t>(S) * H * 2) * 2;      // dy_w, dx_slot
      b += round256(static_cast<size_t>(S) * 2 * I * 2);      // dG
      b += round256(static_cast<size_t>(S) * I * 2);          // dh
      b += round256(static_cast<size_t>(S) * 4) * 2;          // dgates, unit weights
      b += round256(static_cast<size_t>(E + 1) * 4);          // padded segment starts
      // the transposed, expert-padded operands of one weight gradient at a time
      b += round256(static_cast<size_t>(2 * I + H > H + I ? 2 * I + H : H + I) *
                    wgrad_pad_cols(S, E) * 2);
      return b;
    }
    case MOE_OP_FORWARD: {
      size_t b = 0;
      b += round256(static_cast<size_t>(S) * 4);                       // topk_idx
      b += round256(static_cast<size_t>(S) * 4);                       // topk_w
      b += round256(static_cast<size_t>(E + 1) * 4);                   // offsets
      b += round256(static_cast<size_t>(S) * 4) * 2;                   // perm_src, slot_of
      b += round256(static_cast<size_t>(S) * H * act_bytes(act));      // x_perm
      if (act == MOE_E4M3) b += round256(static_cast<size_t>(S) * (H / 128) * 4);
      b += dispatch_ws_bytes(T, E);
      b += h_bytes(S, I, act);
      b += round256(static_cast<size_t>(S) * H * (act == MOE_F32 ? 4 : 2));  // y
      b += 256;                                                               // grid barrier
      return b;
    }
    default:
      return 0;
  }
}

moe_status moe_get_device_error(cudaStream_t stream, int* site) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int host[2] = {0, 0};
  if (cudaMemcpyFromSymbol(host, g_error_word, sizeof(host)) != cudaSuccess) return MOE_ERR_CUDA;
  if (host[0] != 0) {
    const int zero[2] = {0, 0};  // status and site only; the wait limit stays
    if (cudaMemcpyToSymbol(g_error_word, zero, sizeof(zero)) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (site) *site = host[1];
  return static_cast<moe_status>(host[0]);
}

// Checks a routing configuration; fills in the plain router for NULL.
static moe_status check_groups(const moe_router_groups* g, int E, int k, moe_router_groups* out) {
  *out = moe_router_groups{1, 1, 1.0f};
  if (g == nullptr) return MOE_OK;
  if (g->n_group < 1 || g->topk_group < 1 || g->topk_group > g->n_group) return MOE_ERR_INVALID_ARG;
  if (!(g->scale == g->scale) || g->scale == INFINITY || g->scale == -INFINITY)
    return MOE_ERR_INVALID_ARG;
  if (g->n_group > 1) {
    if (E % g->n_group != 0 || (E / g->n_group) % 32 != 0) return MOE_ERR_UNSUPPORTED;
    if (k > g->topk_group * (E / g->n_group)) return MOE_ERR_INVALID_ARG;
  }
  *out = *g;
  return MOE_OK;
}

moe_status moe_route(const float* logits, const float* bias, int T, int E, int k, int score,
                     int renorm, int32_t* topk_idx, float* topk_w, cudaStream_t stream) {
  return moe_route_ex(logits, bias, T, E, k, score, renorm, nullptr, topk_idx, topk_w, stream);
}

moe_status moe_route_ex(const float* logits, const float* bias, int T, int E, int k, int score,
                        int renorm, const moe_router_groups* groups, int32_t* topk_idx,
                        float* topk_w, cudaStream_t stream) {
  if (logits == nullptr || topk_idx == nullptr || topk_w == nullptr) return MOE_ERR_INVALID_ARG;
  if (T < 1 || E < 1 || k < 1) return MOE_ERR_INVALID_ARG;
  if (score != MOE_SCORE_SOFTMAX && score != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (E > 1024 || k > 32 || k > E || !slots_fit(T, k)) return MOE_ERR_UNSUPPORTED;
  if (!aligned(logits, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) ||
      (bias && !aligned(bias, 4)))
    return MOE_ERR_MISALIGNED;
  moe_router_groups g;
  const moe_status gs = check_groups(groups, E, k, &g);
  if (gs != MOE_OK) return gs;
  return cuda_status(launch_route(logits, score == MOE_SCORE_SIGMOID ? bias : nullptr, T, E, k,
                                  score, renorm != 0, topk_idx, topk_w, stream, g.n_group,
                                  g.topk_group, g.scale));
}

moe_status moe_dispatch(const void* x, const float* x_scales, int act, int T, int H, int E, int k,
                        const int32_t* topk_idx, void* x_perm, float* x_perm_scales,
                        int32_t* expert_offsets, int32_t* perm_src, int32_t* slot_of, void* ws,
                        size_t ws_bytes, cudaStream_t stream) {
  moe_status st = check_shapes(T, H, E, k);
  if (st != MOE_OK) return st;
  if (act != MOE_F32 && act != MOE_BF16 && act != MOE_E4M3) return MOE_ERR_INVALID_ARG;
  if (!x || !topk_idx || !x_perm || !expert_offsets || !perm_src || !slot_of)
    return MOE_ERR_INVALID_ARG;
  if (act == MOE_E4M3 && (!x_scales || !x_perm_scales)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(topk_idx, 4) ||
      !aligned(expert_offsets, 4) || !aligned(perm_src, 4) || !aligned(slot_of, 4))
    return MOE_ERR_MISALIGNED;
  if (act == MOE_E4M3 && (!aligned(x_scales, 4) || !aligned(x_perm_scales, 4)))
    return MOE_ERR_MISALIGNED;
  if (!ws || !aligned(ws, 256) || ws_bytes < dispatch_ws_bytes(T, E)) return MOE_ERR_WORKSPACE;
  const int row_bytes = H * static_cast<int>(act_bytes(act));
  return cuda_status(launch_dispatch(x, act == MOE_E4M3 ? x_scales : nullptr, row_bytes, T, H, E,
                                     k, topk_idx, x_perm, x_perm_scales, expert_offsets,
                                     perm_src, slot_of, ws, stream));
}

moe_status moe_dispatch_quant(const void* x, int T, int H, int E, int k,
                              const int32_t* topk_idx, void* x_perm, float* x_perm_scales,
                              int32_t* expert_offsets, int32_t* perm_src, int32_t* slot_of,
                              void* ws, size_t ws_bytes, cudaStream_t stream) {
  moe_status st = check_shapes(T, H, E, k);
  if (st != MOE_OK) return st;
  if (!x || !topk_idx || !x_perm || !x_perm_scales || !expert_offsets || !perm_src || !slot_of)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(x_perm_scales, 4) ||
      !aligned(topk_idx, 4) || !aligned(expert_offsets, 4) || !aligned(perm_src, 4) ||
      !aligned(slot_of, 4))
    return MOE_ERR_MISALIGNED;
  if (!ws || !aligned(ws, 256) || ws_bytes < dispatch_ws_bytes(T, E)) return MOE_ERR_WORKSPACE;
  return cuda_status(launch_dispatch(x, nullptr, H, T, H, E, k, topk_idx, x_perm, x_perm_scales,
                                     expert_offsets, perm_src, slot_of, ws, stream, true));
}

static moe_status check_ffn(const void* a, const float* a_scales, const int32_t* offsets, int S,
                            int H, int I, int E, const moe_weights* W, const void* out) {
  if (!a || !offsets || !out) return MOE_ERR_INVALID_ARG;
  if (S < 1 || H < 128 || I < 128 || E < 1) return MOE_ERR_INVALID_ARG;
  if (H % 128 != 0 || I % 128 != 0 || E > 1024) return MOE_ERR_UNSUPPORTED;
  moe_status st = check_weights(W, -1);
  if (st != MOE_OK) return st;
  if (W->act == MOE_E4M3 && !a_scales) return MOE_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(out, 16) || !aligned(offsets, 4)) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

moe_status moe_expert_linear1(const void* x_perm, const float* x_perm_scales,
                              const int32_t* expert_offsets, int S, int H, int I, int E,
                              const moe_weights* W, void* h, float* h_scales, void* ws,
                              size_t ws_bytes, cudaStream_t stream) {
  (void)ws;
  (void)ws_bytes;
  moe_status st = check_ffn(x_perm, x_perm_scales, expert_offsets, S, H, I, E, W, h);
  if (st != MOE_OK) return st;
  if (W->act == MOE_E4M3 && !h_scales) return MOE_ERR_INVALID_ARG;
  FfnArgs a{W->act, W->wt, x_perm, x_perm_scales, expert_offsets, S, H, I, E,
            W->w1, W->w1_scales, h, h_scales, device_error_word(), W->scale_fmt};
  return run_ffn(1, a, stream);
}

moe_status moe_expert_linear2(const void* h, const float* h_scales, const int32_t* expert_offsets,
                              int S, int H, int I, int E, const moe_weights* W, void* y, void* ws,
                              size_t ws_bytes, cudaStream_t stream) {
  (void)ws;
  (void)ws_bytes;
  moe_status st = check_ffn(h, h_scales, expert_offsets, S, H, I, E, W, y);
  if (st != MOE_OK) return st;
  FfnArgs a{W->act, W->wt, h, h_scales, expert_offsets, S, H, I, E,
            W->w2, W->w2_scales, y, nullptr, device_error_word(), W->scale_fmt};
  return run_ffn(2, a, stream);
}

moe_status moe_fused_ffn(const void* x_perm, const float* x_perm_scales,
                         const int32_t* expert_offsets, int S, int H, int I, int E,
                         const moe_weights* W, void* y, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  moe_status st = check_ffn(x_perm, x_perm_scales, expert_offsets, S, H, I, E, W, y);
  if (st != MOE_OK) return st;
  const size_t need = h_bytes(S, I, W->act);
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return MOE_ERR_WORKSPACE;
  char* p = static_cast<char*>(ws);
  void* h = p;
  float* hs = W->act == MOE_E4M3
                  ? reinterpret_cast<float*>(p + round256(static_cast<size_t>(S) * I * act_bytes(W->act)))
                  : nullptr;
  st = moe_expert_linear1(x_perm, x_perm_scales, expert_offsets, S, H, I, E, W, h, hs, nullptr, 0,
                          stream);
  if (st != MOE_OK) return st;
  return moe_expert_linear2(h, hs, expert_offsets, S, H, I, E, W, y, nullptr, 0, stream);
}

moe_status moe_combine(const void* y, int y_dt, const int32_t* slot_of, const float* topk_w,
                       int T, int k, int H, void* out, int out_dt, cudaStream_t stream) {
  if (!y || !slot_of || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  if (T < 1 || k < 1 || H < 8) return MOE_ERR_INVALID_ARG;
  if (k > 32 || H % 8 != 0 || !slots_fit(T, k)) return MOE_ERR_UNSUPPORTED;
  if ((y_dt != MOE_F32 && y_dt != MOE_BF16) || (out_dt != MOE_F32 && out_dt != MOE_BF16))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(y, 16) || !aligned(out, 16) || !aligned(slot_of, 4) || !aligned(topk_w, 4))
    return MOE_ERR_MISALIGNED;
  return cuda_status(launch_combine(y, y_dt == MOE_F32, slot_of, topk_w, T, k, H, out,
                                    out_dt == MOE_F32, stream));
}

moe_status moe_forward(const void* x, const float* x_scales, const float* logits,
                       const float* bias, int score, int renorm, int T, int H, int E, int k,
                       int I, const moe_weights* W, void* out, int32_t* topk_idx_out,
                       float* topk_w_out, int32_t* offsets_out, void* ws, size_t ws_bytes,
                       cudaStream_t stream) {
  return moe_forward_ex(x, x_scales, logits, bias, score, renorm, nullptr, T, H, E, k, I, W, out,
                        topk_idx_out, topk_w_out, offsets_out, ws, ws_bytes, stream);
}

moe_status moe_forward_ex(const void* x, const float* x_scales, const float* logits,
                          const float* bias, int score, int renorm,
                          const moe_router_groups* groups, int T, int H, int E, int k, int I,
                          const moe_weights* W, void* out, int32_t* topk_idx_out,
                          float* topk_w_out, int32_t* offsets_out, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
  moe_status st = check_shapes(T, H, E, k);
  if (st != MOE_OK) return st;
  moe_router_groups rg;
  st = check_groups(groups, E, k, &rg);
  if (st != MOE_OK) return st;
  if (I < 128) return MOE_ERR_INVALID_ARG;
  if (I % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (!x || !logits || !out) return MOE_ERR_INVALID_ARG;
  st = check_weights(W, -1);
  if (st != MOE_OK) return st;
  const int act = W->act;
  // E4M3 activations without x_scales: x is BF16 and the dispatch quantises it
  const size_t need = moe_workspace_size(MOE_OP_FORWARD, T, H, E, k, I, act, W->wt);
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return MOE_ERR_WORKSPACE;
  const int S = T * k;
  char* p = static_cast<char*>(ws);
  auto take = [&](size_t bytes) {
    char* r = p;
    p += round256(bytes);
    return r;
  };
  int32_t* topk_idx = reinterpret_cast<int32_t*>(take(static_cast<size_t>(S) * 4));
  float* topk_w = reinterpret_cast<float*>(take(static_cast<size_t>(S) * 4));
  int32_t* offsets = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E + 1) * 4));
  int32_t* perm_src = reinterpret_cast<int32_t*>(take(static_cast<size_t>(S) * 4));
  int32_t* slot_of = reinterpret_cast<int32_t*>(take(static_cast<size_t>(S) * 4));
  void* x_perm = take(static_cast<size_t>(S) * H * act_bytes(act));
  float* x_perm_scales =
      act == MOE_E4M3 ? reinterpret_cast<float*>(take(static_cast<size_t>(S) * (H / 128) * 4))
                      : nullptr;
  void* dws = take(dispatch_ws_bytes(T, E));
  void* ffn_ws = take(h_bytes(S, I, act));
  void* y = take(static_cast<size_t>(S) * H * (act == MOE_F32 ? 4 : 2));
  uint32_t* bar = reinterpret_cast<uint32_t*>(take(256));
  if (topk_idx_out) topk_idx = topk_idx_out;
  if (topk_w_out) topk_w = topk_w_out;
  if (offsets_out) offsets = offsets_out;

  if (act != MOE_F32 && W->scale_fmt == MOE_SCALE_POW2) {
    // tensor-core formats with power-of-two scales: the whole layer in one persistent launch
    if (!aligned(logits, 4) || (bias && !aligned(bias, 4)) || !aligned(out, 16) ||
        !aligned(x, 16) || (x_scales && !aligned(x_scales, 4)))
      return MOE_ERR_MISALIGNED;
    if (score != MOE_SCORE_SOFTMAX && score != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
    const size_t hsz = round256(static_cast<size_t>(S) * I * act_bytes(act));
    ForwardArgs fa;
    fa.x = x;
    fa.x_scales = act == MOE_E4M3 ? x_scales : nullptr;
    fa.logits = logits;
    fa.bias = score == MOE_SCORE_SIGMOID ? bias : nullptr;
    fa.sigmoid = score == MOE_SCORE_SIGMOID;
    fa.renorm = renorm != 0;
    fa.n_group = rg.n_group;
    fa.topk_group = rg.topk_group;
    fa.scale = rg.scale;
    fa.T = T;
    fa.H = H;
    fa.E = E;
    fa.k = k;
    fa.I = I;
    fa.act = act;
    fa.wt = W->wt;
    fa.w1 = W->w1;
    fa.w1_scales = W->w1_scales;
    fa.w2 = W->w2;
    fa.w2_scales = W->w2_scales;
    fa.topk_idx = topk_idx;
    fa.topk_w = topk_w;
    fa.offsets = offsets;
    fa.perm_src = perm_src;
    fa.slot_of = slot_of;
    fa.x_perm = x_perm;
    fa.x_perm_scales = x_perm_scales;
    fa.cnt = static_cast<int32_t*>(dws);
    fa.totals = reinterpret_cast<int32_t*>(
        static_cast<char*>(dws) + round256(static_cast<size_t>((T + kChunkTokens - 1) / kChunkTokens) * E * 4));
    fa.h = ffn_ws;
    fa.h_scales = act == MOE_E4M3 ? reinterpret_cast<float*>(static_cast<char*>(ffn_ws) + hsz) : nullptr;
    fa.y = y;
    fa.out = out;
    fa.bar = bar;
    fa.err = device_error_word();
    return cuda_status(launch_forward_fused(fa, stream));
  }

  st = moe_route_ex(logits, bias, T, E, k, score, renorm, &rg, topk_idx, topk_w, stream);
  if (st != MOE_OK) return st;
  st = moe_dispatch(x, x_scales, act, T, H, E, k, topk_idx, x_perm, x_perm_scales, offsets,
                    perm_src, slot_of, dws, dispatch_ws_bytes(T, E), stream);
  if (st != MOE_OK) return st;
  st = moe_fused_ffn(x_perm, x_perm_scales, offsets, S, H, I, E, W, y, ffn_ws, h_bytes(S, I, act),
                     stream);
  if (st != MOE_OK) return st;
  const int ydt = act == MOE_F32 ? MOE_F32 : MOE_BF16;
  return moe_combine(y, ydt, slot_of, topk_w, T, k, H, out, ydt, stream);
}

moe_status moe_transpose_experts(const void* src, int dtype, int E, int R, int C, void* dst,
                                 cudaStream_t stream) {
  if (!src || !dst || E < 1 || R < 1 || C < 1) return MOE_ERR_INVALID_ARG;
  int eb = 0;
  switch (dtype) {
    case MOE_F32: eb = 4; break;
    case MOE_BF16: eb = 2; break;
    case MOE_E4M3: eb = 1; break;
    case MOE_E2M1: return MOE_ERR_UNSUPPORTED;
    default: return MOE_ERR_INVALID_ARG;
  }
  if (E > 65535 || (R + 31) / 32 > 65535) return MOE_ERR_UNSUPPORTED;  // grid limits
  if (!aligned(src, eb) || !aligned(dst, eb)) return MOE_ERR_MISALIGNED;
  const uintptr_t n = static_cast<uintptr_t>(E) * R * C * eb;
  const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), d0 = reinterpret_cast<uintptr_t>(dst);
  if (s0 < d0 + n && d0 < s0 + n) return MOE_ERR_INVALID_ARG;  // overlapping buffers
  return cuda_status(launch_transpose(src, eb, E, R, C, dst, stream));
}

moe_status moe_expert_backward(const moe_backward_args* a, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
  if (a == nullptr) return MOE_ERR_INVALID_ARG;
  moe_status st = check_shapes(a->T, a->H, a->E, a->k);
  if (st != MOE_OK) return st;
  if (a->I < 128) return MOE_ERR_INVALID_ARG;
  if (a->I % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (a->score != MOE_SCORE_SOFTMAX && a->score != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (!(a->scale == a->scale) || a->scale == INFINITY || a->scale == -INFINITY)
    return MOE_ERR_INVALID_ARG;
  const void* bf[] = {a->dout, a->x_perm, a->h, a->y, a->w1, a->w1_t, a->w2_t, a->dx,
                      a->dw1, a->dw2};
  for (const void* q : bf) {
    if (q == nullptr) return MOE_ERR_INVALID_ARG;
    if (!aligned(q, 16)) return MOE_ERR_MISALIGNED;
  }
  const void* w4[] = {a->logits, a->topk_idx, a->topk_w, a->expert_offsets, a->slot_of,
                      a->dlogits};
  for (const void* q : w4) {
    if (q == nullptr) return MOE_ERR_INVALID_ARG;
    if (!aligned(q, 4)) return MOE_ERR_MISALIGNED;
  }
  const int T = a->T, H = a->H, E = a->E, k = a->k, I = a->I, S = T * k;
  const size_t need = moe_workspace_size(MOE_OP_BACKWARD, T, H, E, k, I, MOE_BF16, MOE_BF16);
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return MOE_ERR_WORKSPACE;
  char* p = static_cast<char*>(ws);
  auto take = [&p](size_t bytes) {
    void* q = p;
    p += round256(bytes);
    return q;
  };
  void* dy_w = take(static_cast<size_t>(S) * H * 2);
  void* dx_slot = take(static_cast<size_t>(S) * H * 2);
  void* dG = take(static_cast<size_t>(S) * 2 * I * 2);
  void* dh = take(static_cast<size_t>(S) * I * 2);
  float* dgates = static_cast<float*>(take(static_cast<size_t>(S) * 4));
  float* ones = static_cast<float*>(take(static_cast<size_t>(S) * 4));
  int32_t* pk = static_cast<int32_t*>(take(static_cast<size_t>(E + 1) * 4));
  const size_t Kp = wgrad_pad_cols(S, E);
  char* tbuf = static_cast<char*>(take(static_cast<size_t>(2 * I + H > H + I ? 2 * I + H : H + I) * Kp * 2));
  int* err = device_error_word();
  // combine and router backward
  if (launch_combine_backward(a->dout, a->y, a->slot_of, a->topk_w, T, k, H, dy_w, dgates,
                              stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (launch_gate_backward(a->logits, a->topk_idx, dgates, T, E, k,
                           a->score == MOE_SCORE_SIGMOID, a->renorm != 0, a->scale, a->dlogits,
                           stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  // expert GEMM of the forward pass, out[S, N] = A[S, K] . W[E, N, K]^T: FfnArgs with
  // I = K and H = N (its linear-2 form).  dh = dy_w . W2 first; then linear-1 in its backward
  // form recomputes the pre-activations and turns them and dh into dG in its epilogue
  const FfnArgs dh_args{MOE_BF16, MOE_BF16, dy_w, nullptr, a->expert_offsets, S, I, H,
                        E, a->w2_t, nullptr, dh, nullptr, err};
  if (launch_linear2_tc(dh_args, stream) != cudaSuccess) return MOE_ERR_CUDA;
  FfnArgs dg_args{MOE_BF16, MOE_BF16, a->x_perm, nullptr, a->expert_offsets, S, H, I,
                  E, a->w1, nullptr, dG, nullptr, err};
  dg_args.dh = dh;
  if (launch_linear1_dgate_tc(dg_args, stream) != cudaSuccess) return MOE_ERR_CUDA;
  const FfnArgs dx_args{MOE_BF16, MOE_BF16, dG, nullptr, a->expert_offsets, S, H, 2 * I,
                        E, a->w1_t, nullptr, dx_slot, nullptr, err};
  if (launch_linear2_tc(dx_args, stream) != cudaSuccess) return MOE_ERR_CUDA;
  // dx[t] = sum of the token's slot rows (the combine with unit weights)
  if (launch_fill(ones, static_cast<size_t>(S), 1.0f, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (launch_combine(dx_slot, 0, a->slot_of, ones, T, k, H, a->dx, 0, stream) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  // weight gradients on tensor cores: both operands transposed into expert-padded copies
  // (dG^T [2I, Kp] and x^T [H, Kp], then dy_w^T [H, Kp] and h^T [I, Kp], one pair at a time)
  const int32_t* offs = a->expert_offsets;
  void* at = tbuf;
  if (launch_wgrad_pad_offsets(offs, E, pk, stream) != cudaSuccess) return MOE_ERR_CUDA;
  void* bt = tbuf + static_cast<size_t>(2 * I) * Kp * 2;
  if (launch_pad_transpose(dG, S, 2 * I, offs, pk, E, at, stream) != cudaSuccess ||
      launch_pad_transpose(a->x_perm, S, H, offs, pk, E, bt, stream) != cudaSuccess ||
      launch_wgrad_tc(at, bt, offs, pk, S, E, 2 * I, H, a->dw1, err, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  bt = tbuf + static_cast<size_t>(H) * Kp * 2;
  if (launch_pad_transpose(dy_w, S, H, offs, pk, E, at, stream) != cudaSuccess ||
      launch_pad_transpose(a->h, S, I, offs, pk, E, bt, stream) != cudaSuccess ||
      launch_wgrad_tc(at, bt, offs, pk, S, E, H, I, a->dw2, err, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"
