"""Backward of the MoE expert layer in fp64 (oracle; test infrastructure only).

The gradients of the layer's plain definition

    out[t] = sum_{j<k} w[t, j] * W2_e . SwiGLU(W1_e . x_t),   e = topk_idx[t, j],

evaluated in fp64 on the dequantised inputs.  Sources: youleyou, "DeepSeek 模型更新解读
Tile Kernels 与 DeepEP V2 新特性", section "Tile Kernels：逼近硬件极限的底层优化", feature
list, model-layer item (autograd wrappers that turn the kernels into trainable layers);
setupai, "DeepSeek 更新 DeepGEMM 支援 Mega MoE", key points (distributed training); the
forward steps follow oracle.moe.

Readings (the pages give no backward formulas):
* The top-k selection is piecewise constant in the logits and carries no gradient; the
  gates do, through the router's gate function (softmax over the selected logits, the full
  softmax without renormalisation, or the renormalised sigmoid).  The sigmoid router's
  selection bias enters the selection only, so its gradient is zero.
* Storage roundings of the forward (h, y, out, the quantised formats) are not
  differentiated: this is the gradient of the fp64 function on the dequantised values
  (straight through every rounding).
* The routed scaling factor multiplies every gate and so every gate gradient.

Each function states the derivative it evaluates; none of them is blocked, fused or
reordered beyond the plain matrix products.
"""
from __future__ import annotations

import numpy as np

from .moe import Layer, dispatch, route


def _sigmoid(v: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-v))


def swiglu_grad(gate: np.ndarray, up: np.ndarray, dh: np.ndarray):
    """h = silu(g) * u with silu(g) = g * sigma(g).

    dh/dg = u * sigma(g) * (1 + g * (1 - sigma(g))),  dh/du = silu(g).
    Returns (dgate, dup) for the upstream gradient dh."""
    s = _sigmoid(gate)
    return dh * up * s * (1.0 + gate * (1.0 - s)), dh * gate * s


def expert_ffn_exact(x: np.ndarray, w1: np.ndarray, w2: np.ndarray):
    """y = W2 . SwiGLU(W1 . x) in fp64 with no storage rounding; also returns gate, up, h."""
    I = w1.shape[0] // 2
    gate = x @ w1[:I].T
    up = x @ w1[I:].T
    h = gate * _sigmoid(gate) * up
    return h @ w2.T, gate, up, h


def expert_ffn_grad(x: np.ndarray, w1: np.ndarray, w2: np.ndarray, dy: np.ndarray):
    """Gradients of y = W2 . SwiGLU(W1 . x) for one expert's rows.

    x [n, H], w1 [2I, H] (rows [0, I) gate, [I, 2I) up), w2 [H, I], dy [n, H].
    dh = dy W2;  dW2 = dy^T h;  (dgate, dup) = swiglu_grad;  dW1 = [dgate^T x; dup^T x];
    dx = dgate W1_gate + dup W1_up.   Returns (dx, dw1, dw2)."""
    I = w1.shape[0] // 2
    _, gate, up, h = expert_ffn_exact(x, w1, w2)
    dh = dy @ w2
    dgate, dup = swiglu_grad(gate, up, dh)
    dw1 = np.concatenate([dgate.T @ x, dup.T @ x], axis=0)
    dw2 = dy.T @ h
    dx = dgate @ w1[:I] + dup @ w1[I:]
    return dx, dw1, dw2


def gate_grad(logits, topk_idx, dw, score: str, renorm: bool = True, scale: float = 1.0):
    """d loss / d logits from d loss / d gates (dw [T, k]), the selection held fixed.

    softmax, renorm:    p = softmax over the selected logits, w = scale * p;
                        dl_j = scale * p_j * (dw_j - sum_i p_i dw_i) for selected j, else 0.
    softmax, no renorm: p = softmax over all E logits, w_j = scale * p_{e_j};
                        dl_m = scale * p_m * ([m selected] dw_m - sum_j p_{e_j} dw_j).
    sigmoid, renorm:    s = sigma(l), w_j = scale * s_j / sum_sel s;
                        dl_j = scale * (dw_j - sum_i (s_i / sum_sel s) dw_i) / sum_sel s
                               * s_j (1 - s_j) for selected j, else 0.
    sigmoid, no renorm: dl_j = scale * dw_j * s_j (1 - s_j) for selected j, else 0."""
    l = np.asarray(logits, np.float64)
    idx = np.asarray(topk_idx, np.int64)
    dw = np.asarray(dw, np.float64)
    T, E = l.shape
    rows = np.arange(T)[:, None]
    dl = np.zeros((T, E), np.float64)
    sel = l[rows, idx]
    if score == "softmax":
        if renorm:
            z = np.exp(sel - sel.max(axis=1, keepdims=True))
            p = z / z.sum(axis=1, keepdims=True)
            dl[rows, idx] = scale * p * (dw - (p * dw).sum(axis=1, keepdims=True))
        else:
            z = np.exp(l - l.max(axis=1, keepdims=True))
            pall = z / z.sum(axis=1, keepdims=True)
            psel = pall[rows, idx]
            dl = -scale * pall * (psel * dw).sum(axis=1, keepdims=True)
            dl[rows, idx] += scale * psel * dw
    elif score == "sigmoid":
        s = _sigmoid(sel)
        if renorm:
            tot = s.sum(axis=1, keepdims=True)
            q = s / tot
            ds = (dw - (q * dw).sum(axis=1, keepdims=True)) / tot
        else:
            ds = dw
        dl[rows, idx] = scale * ds * s * (1.0 - s)
    else:
        raise ValueError(score)
    return dl


def _routing(logits, bias, k, score, renorm, n_group, topk_group, scale):
    """Selection as the forward makes it (on the fp32 logits); gates recomputed in fp64 from
    the logits as given."""
    idx, _ = route(logits, bias, k, score, renorm, n_group, topk_group, scale)
    l = np.asarray(logits, np.float64)
    rows = np.arange(l.shape[0])[:, None]
    sel = l[rows, idx]
    if score == "softmax":
        if renorm:
            z = np.exp(sel - sel.max(axis=1, keepdims=True))
            w = z / z.sum(axis=1, keepdims=True)
        else:
            z = np.exp(l - l.max(axis=1, keepdims=True))
            w = (z / z.sum(axis=1, keepdims=True))[rows, idx]
    else:
        s = _sigmoid(sel)
        w = s / s.sum(axis=1, keepdims=True) if renorm else s
    return idx, w * scale


def forward_values(x, logits, bias, w1, w2, k: int, score: str, renorm: bool = True,
                   n_group: int = 1, topk_group: int = 0, scale: float = 1.0):
    """The layer in fp64 with no storage rounding, on fp64 values: x [T, H], w1 [E, 2I, H],
    w2 [E, H, I].  This is the function backward_values differentiates.  Returns out [T, H]."""
    x = np.asarray(x, np.float64)
    idx, w = _routing(logits, bias, k, score, renorm, n_group, topk_group, scale)
    out = np.zeros_like(x)
    for e in np.unique(idx):
        rr, jj = np.nonzero(idx == e)
        y, _, _, _ = expert_ffn_exact(x[rr], w1[e], w2[e])
        np.add.at(out, rr, w[rr, jj][:, None] * y)
    return out


def backward_values(x, logits, bias, w1, w2, k: int, score: str, dout, renorm: bool = True,
                    n_group: int = 1, topk_group: int = 0, scale: float = 1.0):
    """Gradients of sum(dout * forward_values(...)) with respect to x, w1, w2 and the logits.

    Per slot (t, j) routed to e: y_tj = W2_e . SwiGLU(W1_e . x_t);
      d loss / d w[t, j] = dout[t] . y_tj,   d loss / d y_tj = w[t, j] * dout[t];
    the slot's expert gradients (expert_ffn_grad) are summed over the expert's slots into
    dW1_e, dW2_e and over a token's k slots into dx[t]; the gate gradients go through
    gate_grad.  Experts no token picked get zero gradients; so does the selection bias.

    Returns dict(dx [T, H], dw1 [E, 2I, H], dw2 [E, H, I], dlogits [T, E], dbias [E] or
    None, topk_idx, offsets)."""
    x = np.asarray(x, np.float64)
    dout = np.asarray(dout, np.float64)
    E = np.asarray(logits).shape[1]
    idx, w = _routing(logits, bias, k, score, renorm, n_group, topk_group, scale)
    _, offsets, perm_src, _ = dispatch(idx, E)
    tok = perm_src // k
    rank = perm_src % k
    dx = np.zeros_like(x)
    dgates = np.zeros_like(w)
    dw1 = np.zeros(np.shape(w1), np.float64)
    dw2 = np.zeros(np.shape(w2), np.float64)
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        t, j = tok[a:b], rank[a:b]
        y, _, _, _ = expert_ffn_exact(x[t], w1[e], w2[e])
        dgates[t, j] = np.einsum("nh,nh->n", dout[t], y)
        dxe, dw1[e], dw2[e] = expert_ffn_grad(x[t], w1[e], w2[e], w[t, j][:, None] * dout[t])
        np.add.at(dx, t, dxe)
    dl = gate_grad(logits, idx, dgates, score, renorm, scale)
    dbias = None if bias is None else np.zeros(E, np.float64)
    return dict(dx=dx, dw1=dw1, dw2=dw2, dlogits=dl, dbias=dbias, topk_idx=idx,
                offsets=offsets)


def _weights_f64(L: Layer):
    pairs = [L.expert_weights(e) for e in range(L.E)]
    return np.stack([p[0] for p in pairs]), np.stack([p[1] for p in pairs])


def forward_exact(L: Layer, n_group: int = 1, topk_group: int = 0, scale: float = 1.0):
    """forward_values on the layer's dequantised input and weights."""
    w1, w2 = _weights_f64(L)
    return forward_values(L.x_hat(), L.logits, L.bias, w1, w2, L.k, L.score, L.renorm,
                          n_group, topk_group, scale)


def layer_backward(L: Layer, dout, n_group: int = 1, topk_group: int = 0, scale: float = 1.0):
    """backward_values on the layer's dequantised input and weights (the gradients with
    respect to the dequantised values, straight through the formats)."""
    w1, w2 = _weights_f64(L)
    return backward_values(L.x_hat(), L.logits, L.bias, w1, w2, L.k, L.score, dout, L.renorm,
                           n_group, topk_group, scale)


def layer_backward_stored(L: Layer, dout, store=None, return_slots=False):
    """The backward of a BF16 layer with every intermediate stored where the CUDA path stores
    it (`store` rounds a value to its storage format; default BF16 round-to-nearest-even):

      forward tensors, as the forward pass stores them:
        h = store(silu(g) * u),  y = store(h W2^T),  gates w as fp32
      dgates[t, j] = dout[t] . y[slot(t, j)]         (an fp32 result: kept exact here)
      dy_w[slot]   = store(w[t, j] * dout[t])
      dh           = store(dy_w W2)
      dG           = store(swiglu_grad(g, u, dh))     (gate and up halves; the
                                                       pre-activations g, u = x W1^T
                                                       are recomputed, not stored)
      dx_slot      = store(dG W1),   dx[t] = store(sum over the token's slots of dx_slot)
      dW1_e = dG_e^T x_e,  dW2_e = dy_w,e^T h_e        (fp32 results: exact here)
      dlogits      = gate_grad(dgates)                (an fp32 result)

    With store = identity this is layer_backward up to the fp32 storage of the gates.
    Returns the same dict as layer_backward; with return_slots, also "slots": the stored
    per-slot values the weight gradients sum (dG, x, dy_w, h) and dh, rows in dispatch
    order."""
    from .formats import round_bf16
    st = round_bf16 if store is None else store
    dout = np.asarray(dout, np.float64)
    idx, w = route(L.logits, L.bias, L.k, L.score, L.renorm)
    w32 = w.astype(np.float32).astype(np.float64)
    _, offsets, perm_src, _ = dispatch(idx, L.E)
    tok = perm_src // L.k
    rank = perm_src % L.k
    xh = L.x_hat()
    T, H = xh.shape
    dx_slot = np.zeros((tok.size, H), np.float64)
    slots = {}
    dgates = np.zeros_like(w)
    dw1 = dw2 = None
    for e in range(L.E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        w1, w2 = L.expert_weights(e)
        if dw1 is None:
            dw1 = np.zeros((L.E,) + w1.shape, np.float64)
            dw2 = np.zeros((L.E,) + w2.shape, np.float64)
        if a == b:
            continue
        t, j = tok[a:b], rank[a:b]
        x = xh[t]
        _, gate, up, _ = expert_ffn_exact(x, w1, w2)
        h = st(gate * _sigmoid(gate) * up)
        y = st(h @ w2.T)
        dgates[t, j] = np.einsum("nh,nh->n", dout[t], y)
        dyw = st(w32[t, j][:, None] * dout[t])
        dh = st(dyw @ w2)
        dg, du = swiglu_grad(gate, up, dh)
        dG = np.concatenate([st(dg), st(du)], axis=1)
        dx_slot[a:b] = st(dG @ w1)
        dw1[e] = dG.T @ x
        dw2[e] = dyw.T @ h
        if return_slots:
            for n, v in (("dG", dG), ("x", x), ("dy_w", dyw), ("h", h), ("dh", dh)):
                slots.setdefault(n, np.zeros((tok.size, v.shape[1]), np.float64))[a:b] = v
    dx = np.zeros((T, H), np.float64)
    np.add.at(dx, tok, dx_slot)
    dl = gate_grad(L.logits, idx, dgates, L.score, L.renorm)
    dbias = None if L.bias is None else np.zeros(L.E, np.float64)
    res = dict(dx=st(dx), dw1=dw1, dw2=dw2, dlogits=dl, dbias=dbias, topk_idx=idx,
               offsets=offsets)
    if return_slots:
        res["slots"] = slots
    return res
