"""The MoE expert layer, step by step, in fp64 (oracle; test infrastructure only).

Steps and the passages they follow:

1. route     -- youleyou, "DeepSeek 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", section
                "Tile Kernels：逼近硬件极限的底层优化", feature list, gating item (top-k
                expert selection with scoring) and routing item (weight normalisation).
2. dispatch  -- jiqizhixin, "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了", section
                "Mega MoE 是什么？", pipeline paragraph (tokens are first dispatched to the
                experts); youleyou, same feature list, routing item (token-to-expert mapping,
                fused expand).
3. linear-1, SwiGLU, linear-2 -- jiqizhixin, same section, pipeline paragraph (a linear
                layer, the SwiGLU activation, a second linear layer) and the FP8 x FP4
                paragraph; youleyou, feature list, quantisation item (FP8/FP4 per-token and
                per-block quantisation fused with SwiGLU).
4. combine   -- jiqizhixin, same section, pipeline paragraph (results are put back
                together); youleyou, routing item (fused reduce).
0. (before dispatch, for BF16 input to an E4M3 layer) activation quantisation -- youleyou,
                feature list, quantisation item (FP8 per-block quantisation); jiqizhixin,
                FP8 x FP4 paragraph (FP8 activations): quantize_activations.

Tensor formats follow the layer's data contract:
  x      [T, H]   f32 | bf16 bits (uint16) | E4M3 codes (uint8) + x_scales f32 [T, H/128]
  W1     [E, 2I, H]  rows [0, I) gate, [I, 2I) up      (E2M1: packed [E, 2I, H/2])
  W2     [E, H, I]                                     (E2M1: packed [E, H, I/2])
  W scales: E4M3 -> f32 [E, rows/128, cols/128]; E2M1 -> UE8M0 bytes [E, rows, cols/32]
  h      [S, I]   stored as f32 | BF16 | E4M3 with a power-of-two scale per 1x128 block
  y      [S, H]   BF16 (f32 for the f32 layer), unweighted, one row per slot
  out    [T, H]   BF16 (f32 for the f32 layer)
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .fexp import sigmoid_f32
from .formats import (bf16_bits_to_f64, e2m1_decode_packed, e4m3_decode, e4m3_encode,
                      round_bf16, ue8m0_decode)

E4M3_MAX = 448.0


# ----------------------------------------------------------------------------------------
# 1. route
# ----------------------------------------------------------------------------------------
def route(logits, bias, k: int, score: str, renorm: bool = True, n_group: int = 1,
          topk_group: int = 0, scale: float = 1.0):
    """Top-k expert selection and gate weights.

    softmax: keys are the fp32 logits themselves; gates are exp(l_j - m) / sum over the k
             selected (renorm) or over all E experts (no renorm), m the largest logit used.
    sigmoid: s = sigmoid(l) in fp32 (oracle.fexp), keys = fp32(s + b_e); gates are
             s_j / sum of the selected s (renorm) or s_j (no renorm).
    Group-limited selection (n_group > 1): experts form n_group consecutive groups of
    E / n_group; a group's score is the fp32 sum of its two largest keys (its only key when
    a group holds one expert); the topk_group best groups (equal scores -> lower group id)
    are kept and the k experts are chosen among theirs only.  Gates are finally multiplied
    by `scale` (the routed scaling factor; 1 leaves them as they are).
    Order: key descending, equal keys -> lower expert id first.  The k experts are returned
    in that rank order, which is also the order in which the combine sums them.

    Returns (topk_idx int32 [T, k], topk_w fp64 [T, k])."""
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    if score == "softmax":
        keys = logits
    elif score == "sigmoid":
        s = sigmoid_f32(logits)
        b = np.zeros(E, np.float32) if bias is None else np.asarray(bias, np.float32)
        keys = (s + b[None, :]).astype(np.float32)
    else:
        raise ValueError(score)
    rows = np.arange(T)[:, None]
    ids = np.broadcast_to(np.arange(E), (T, E))
    if n_group > 1:
        G = E // n_group
        srt = np.sort(keys.reshape(T, n_group, G), axis=2)
        gscore = srt[:, :, -1] if G == 1 else (srt[:, :, -1] + srt[:, :, -2]).astype(np.float32)
        gorder = np.argsort(-gscore, axis=1, kind="stable")[:, :topk_group]
        allowed = np.zeros((T, n_group), bool)
        allowed[rows, gorder] = True
        allowed = np.repeat(allowed, G, axis=1)
    else:
        allowed = np.ones((T, E), bool)
    # allowed experts first, then key descending, then expert id ascending
    order = np.lexsort((ids, -keys, ~allowed), axis=1)
    idx = order[:, :k].astype(np.int32)
    if score == "softmax":
        l = logits.astype(np.float64)
        sel = l[rows, idx]
        if renorm:
            z = np.exp(sel - sel.max(axis=1, keepdims=True))
            w = z / z.sum(axis=1, keepdims=True)
        else:
            m = l.max(axis=1, keepdims=True)
            w = np.exp(sel - m) / np.exp(l - m).sum(axis=1, keepdims=True)
    else:
        ssel = s.astype(np.float64)[rows, idx]
        w = ssel / ssel.sum(axis=1, keepdims=True) if renorm else ssel
    return idx, w * scale


# ----------------------------------------------------------------------------------------
# 2. dispatch
# ----------------------------------------------------------------------------------------
def dispatch(topk_idx, E: int):
    """Stable counting sort of the T*k (token, rank) pairs by expert.

    Pair (t, j) has flat index t*k + j.  Slots of expert e are
    [offsets[e], offsets[e+1]), holding its tokens in ascending token order (unique, since a
    token selects an expert at most once).
    Returns (counts [E], offsets [E+1], perm_src [S] slot -> t*k+j, slot_of [S] t*k+j -> slot),
    all int32."""
    flat = np.asarray(topk_idx, dtype=np.int64).reshape(-1)
    S = flat.size
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    perm_src = np.argsort(flat, kind="stable")
    slot_of = np.empty(S, np.int64)
    slot_of[perm_src] = np.arange(S)
    return (counts.astype(np.int32), offsets.astype(np.int32), perm_src.astype(np.int32),
            slot_of.astype(np.int32))


# ----------------------------------------------------------------------------------------
# dequantisation
# ----------------------------------------------------------------------------------------
def dequant_x(x, x_scales, act: str) -> np.ndarray:
    """Activations [n, C] -> fp64; E4M3 codes times their 1x128 block scale."""
    if act == "f32":
        return np.asarray(x, np.float32).astype(np.float64)
    if act == "bf16":
        return bf16_bits_to_f64(x)
    if act == "e4m3":
        v = e4m3_decode(x)
        return v * np.repeat(np.asarray(x_scales, np.float64), 128, axis=-1)
    raise ValueError(act)


def dequant_w(w, w_scales, wt: str) -> np.ndarray:
    """One expert's weight matrix [R, C] (E2M1: packed [R, C/2]) -> fp64 [R, C].

    E4M3: code times its 128x128 block scale.  E2M1: code times 2^(b-127) of its 1x32 block."""
    if wt == "f32":
        return np.asarray(w, np.float32).astype(np.float64)
    if wt == "bf16":
        return bf16_bits_to_f64(w)
    if wt == "e4m3":
        s = np.asarray(w_scales, np.float64)
        return e4m3_decode(w) * np.repeat(np.repeat(s, 128, axis=0), 128, axis=1)
    if wt == "e2m1":
        return e2m1_decode_packed(w) * np.repeat(ue8m0_decode(w_scales), 32, axis=1)
    raise ValueError(wt)


# ----------------------------------------------------------------------------------------
# 3. expert FFN
# ----------------------------------------------------------------------------------------
def _pow2_scale_exponent(amax: np.ndarray) -> np.ndarray:
    """Smallest integer n with amax <= 448 * 2^n (n = 0 where amax == 0), but at least -126:
    the scale 2^n is stored as a normal fp32 value (and read as its UE8M0 exponent byte), so
    blocks with amax below 448 * 2^-127 (about 2.6e-36) take 2^-126 and their codes round
    from amax * 2^126 < 224."""
    a = np.asarray(amax, np.float64)
    safe = np.where(a > 0, a, E4M3_MAX)
    n = np.ceil(np.log2(safe / E4M3_MAX)).astype(np.int64)
    # make the defining inequality exact whatever log2 rounded to
    n = np.where(safe > np.ldexp(E4M3_MAX, n), n + 1, n)
    n = np.where(safe <= np.ldexp(E4M3_MAX, n - 1), n - 1, n)
    return np.where(a > 0, np.maximum(n, -126), 0)


def quant_e4m3_1x128(h32):
    """Quantise fp32 rows [n, C] to E4M3 with one power-of-two scale per 1x128 block.

    scale = 2^n, n the smallest integer with amax(block) <= 448 * 2^n; code = nearest E4M3
    of h / scale (ties to even, saturating).  The decision is taken on the fp32 values, the
    precision in which the CUDA epilogue holds h.  Returns (codes u8 [n, C],
    scales f32 [n, C/128])."""
    h32 = np.asarray(h32, np.float32)
    n_rows, C = h32.shape
    blocks = h32.astype(np.float64).reshape(n_rows, C // 128, 128)
    ex = _pow2_scale_exponent(np.abs(blocks).max(axis=2))
    scales = np.ldexp(1.0, ex)
    codes = e4m3_encode(blocks / scales[:, :, None]).reshape(n_rows, C)
    return codes, scales.astype(np.float32)


def quantize_activations(x_bf16_bits):
    """BF16 token rows (uint16 bits [T, H]) -> E4M3 codes [T, H] + fp32 scales [T, H/128],
    one power-of-two scale per 1x128 block by the same rule as h (quant_e4m3_1x128).  BF16
    values are exact in fp32, so the result depends on the input bits alone."""
    x32 = bf16_bits_to_f64(np.asarray(x_bf16_bits, np.uint16)).astype(np.float32)
    return quant_e4m3_1x128(x32)


def _store_h(h: np.ndarray, act: str) -> np.ndarray:
    """Apply h's storage rounding and return the stored value in fp64."""
    if act == "f32":
        return h.astype(np.float32).astype(np.float64)
    if act == "bf16":
        return round_bf16(h)
    if act == "e4m3":
        codes, scales = quant_e4m3_1x128(h.astype(np.float32))
        return dequant_x(codes, scales, "e4m3")
    raise ValueError(act)


def _store_y(y: np.ndarray, act: str) -> np.ndarray:
    return y.astype(np.float32).astype(np.float64) if act == "f32" else round_bf16(y)


def expert_ffn(xh: np.ndarray, w1: np.ndarray, w2: np.ndarray, act: str, return_h=False):
    """One expert on its rows: y = W2 . SwiGLU(W1 . x).

    xh [n, H] fp64 (dequantised), w1 [2I, H], w2 [H, I] fp64.
    gate = x W1[:I]^T, up = x W1[I:]^T, h = silu(gate) * up = gate / (1 + e^-gate) * up,
    h stored in the activation format, y = h_stored W2^T stored as BF16 (f32 layer: fp32)."""
    I = w1.shape[0] // 2
    gate = xh @ w1[:I].T
    up = xh @ w1[I:].T
    with np.errstate(over="ignore"):
        h = gate / (1.0 + np.exp(-gate)) * up
    hs = _store_h(h, act)
    y = _store_y(hs @ w2.T, act)
    return (y, hs) if return_h else y


# ----------------------------------------------------------------------------------------
# 4. combine
# ----------------------------------------------------------------------------------------
def combine(y: np.ndarray, slot_of, topk_w, act: str) -> np.ndarray:
    """out[t] = sum_{j<k} w[t, j] * y[slot_of[t*k + j]], summed in rank order j in fp64,
    then stored as BF16 (f32 layer: fp32).  topk_w is taken as stored (fp32)."""
    w = np.asarray(topk_w, np.float32).astype(np.float64)
    T, k = w.shape
    so = np.asarray(slot_of).reshape(T, k)
    acc = np.zeros((T, y.shape[1]), np.float64)
    for j in range(k):
        acc = acc + w[:, j:j + 1] * y[so[:, j]]
    return _store_y(acc, act)


# ----------------------------------------------------------------------------------------
# end to end
# ----------------------------------------------------------------------------------------
@dataclass
class Layer:
    """Host copies (numpy) of one layer's inputs, in the formats listed in the module doc."""
    act: str
    wt: str
    score: str
    renorm: bool
    k: int
    x: np.ndarray
    x_scales: np.ndarray | None
    logits: np.ndarray
    bias: np.ndarray | None
    w1: np.ndarray
    w1_scales: np.ndarray | None
    w2: np.ndarray
    w2_scales: np.ndarray | None

    @property
    def T(self):
        return self.logits.shape[0]

    @property
    def E(self):
        return self.logits.shape[1]

    def expert_weights(self, e: int):
        s1 = None if self.w1_scales is None else self.w1_scales[e]
        s2 = None if self.w2_scales is None else self.w2_scales[e]
        return dequant_w(self.w1[e], s1, self.wt), dequant_w(self.w2[e], s2, self.wt)

    def x_hat(self, rows=None) -> np.ndarray:
        if rows is None:
            return dequant_x(self.x, self.x_scales, self.act)
        xs = None if self.x_scales is None else self.x_scales[rows]
        return dequant_x(self.x[rows], xs, self.act)


def forward(L: Layer, return_all: bool = False):
    """The whole layer: route -> dispatch -> per-expert FFN -> combine."""
    idx, w = route(L.logits, L.bias, L.k, L.score, L.renorm)
    w32 = w.astype(np.float32)
    counts, offsets, perm_src, slot_of = dispatch(idx, L.E)
    tok = perm_src // L.k
    xh = L.x_hat()
    H = xh.shape[1]
    y = np.zeros((tok.size, H), np.float64)
    h_all = None
    for e in range(L.E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        w1, w2 = L.expert_weights(e)
        ye, he = expert_ffn(xh[tok[a:b]], w1, w2, L.act, return_h=True)
        y[a:b] = ye
        if return_all:
            if h_all is None:
                h_all = np.zeros((tok.size, he.shape[1]), np.float64)
            h_all[a:b] = he
    out = combine(y, slot_of, w32, L.act)
    if not return_all:
        return out
    return dict(out=out, topk_idx=idx, topk_w=w, counts=counts, offsets=offsets,
                perm_src=perm_src, slot_of=slot_of, y=y, h=h_all)


def forward_tokens(L: Layer, tokens, return_y: bool = False):
    """out rows for the listed tokens only (routing is per token, so no other token is
    needed).  Work is grouped by expert so each expert's weights are dequantised once.
    With return_y, also the stored y rows the combine sums, [n, k, H] in rank order, and
    the gates as stored (fp32), [n, k]."""
    tokens = np.asarray(tokens, dtype=np.int64)
    idx, w = route(L.logits[tokens], L.bias, L.k, L.score, L.renorm)
    w32 = w.astype(np.float32).astype(np.float64)
    xh = L.x_hat(tokens)
    acc = [[None] * L.k for _ in range(tokens.size)]
    for e in np.unique(idx):
        rr, jj = np.nonzero(idx == e)
        w1, w2 = L.expert_weights(int(e))
        ye = expert_ffn(xh[rr], w1, w2, L.act)
        for n, (r, j) in enumerate(zip(rr, jj)):
            acc[r][j] = ye[n]
    out = np.zeros((tokens.size, xh.shape[1]), np.float64)
    for r in range(tokens.size):
        for j in range(L.k):
            out[r] = out[r] + w32[r, j] * acc[r][j]
    out = _store_y(out, L.act)
    if return_y:
        return out, np.array([[acc[r][j] for j in range(L.k)] for r in range(tokens.size)]), w32
    return out


def ffn_slots(L: Layer, slots, perm_src, offsets) -> np.ndarray:
    """y rows (stored values, fp64) for the listed dispatch slots."""
    slots = np.asarray(slots, dtype=np.int64)
    offsets = np.asarray(offsets, np.int64)
    experts = np.searchsorted(offsets, slots, side="right") - 1
    tok = np.asarray(perm_src, np.int64)[slots] // L.k
    xh = L.x_hat(tok)
    y = np.zeros((slots.size, xh.shape[1]), np.float64)
    for e in np.unique(experts):
        rr = np.nonzero(experts == e)[0]
        w1, w2 = L.expert_weights(int(e))
        y[rr] = expert_ffn(xh[rr], w1, w2, L.act)
    return y
