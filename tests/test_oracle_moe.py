"""Pins for the oracle's layer steps (CPU only).

Routing: brute force (a full Python sort of all E keys) and special cases (equal logits,
k = E, zero-bias sigmoid = softmax selection).  Dispatch: the invariants of a stable counting
sort.  Combine: it inverts the dispatch.  FFN: with identical experts the layer reduces to one
dense SwiGLU FFN evaluated by torch in fp64; with E = k = 1 it is that FFN exactly; and a
pure-Python brute force (scalar loops, torch casts for the formats) covers every format."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def _layer(wl, dev="cpu"):
    d = synth.to_numpy(synth.make_inputs(wl, dev))
    return oracle.Layer(act=wl.act, wt=wl.wt, score=wl.score, renorm=wl.renorm, k=wl.k,
                        **{n: d[n] for n in ("x", "x_scales", "logits", "bias", "w1",
                                         "w1_scales", "w2", "w2_scales")})


# ---------------------------------------------------------------------------- routing
@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
def test_route_brute_force(score):
    rng = np.random.default_rng(4)
    T, E, k = 40, 13, 4
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[3, :] = 0.25                                   # all tied
    logits[5, 2] = logits[5, 9]                           # one tie
    bias = (rng.standard_normal(E) * 0.1).astype(np.float32)
    idx, w = oracle.route(logits, bias, k, score)
    keys = logits if score == "softmax" else \
        (oracle.sigmoid_f32(logits) + bias[None]).astype(np.float32)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(keys[t, e]), e))
        assert list(idx[t]) == order[:k]
        assert abs(sum(w[t]) - 1) < 1e-12


@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
def test_route_many_ties_brute_force(score):
    # keys drawn from three values: most comparisons are ties, broken by expert id
    rng = np.random.default_rng(11)
    T, E, k = 6, 300, 16
    logits = rng.choice(np.float32([0.0, 0.5, 1.0]), (T, E)).astype(np.float32)
    idx, _ = oracle.route(logits, np.zeros(E, np.float32), k, score)
    keys = logits if score == "softmax" else oracle.sigmoid_f32(logits)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(keys[t, e]), e))
        assert list(idx[t]) == order[:k]


def test_route_equal_logits_special_case():
    logits = np.zeros((3, 8), np.float32)
    for score in ("softmax", "sigmoid"):
        idx, w = oracle.route(logits, None, 3, score)
        assert np.array_equal(idx, np.tile(np.arange(3), (3, 1)))
        assert np.allclose(w, 1 / 3, rtol=0, atol=1e-15)


def test_route_softmax_gates_match_torch():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((20, 16)).astype(np.float32) * 3
    full = torch.softmax(torch.from_numpy(logits).double(), dim=1).numpy()
    # k = E with renorm: gates are the full softmax
    idx, w = oracle.route(logits, None, 16, "softmax", renorm=True)
    assert np.allclose(w, np.take_along_axis(full, idx, 1), rtol=1e-13, atol=0)
    # k < E without renorm: gates are the full-softmax probabilities of the selected experts
    idx, w = oracle.route(logits, None, 5, "softmax", renorm=False)
    assert np.allclose(w, np.take_along_axis(full, idx, 1), rtol=1e-13, atol=0)
    # the selected experts are the five largest probabilities
    assert np.array_equal(np.sort(idx, 1), np.sort(np.argsort(-full, 1)[:, :5], 1))


def test_route_sigmoid_zero_bias_selects_like_softmax():
    # sigmoid is monotone, so with zero bias it selects the same experts as the logits do
    rng = np.random.default_rng(6)
    grid = (np.arange(64) * 0.05 - 1.6).astype(np.float32)   # well separated after sigmoid
    logits = np.stack([rng.permutation(grid) for _ in range(30)])
    i1, _ = oracle.route(logits, np.zeros(64, np.float32), 6, "sigmoid")
    i2, _ = oracle.route(logits, None, 6, "softmax")
    assert np.array_equal(i1, i2)


def test_route_sigmoid_gates():
    rng = np.random.default_rng(7)
    logits = rng.standard_normal((10, 32)).astype(np.float32)
    bias = (rng.standard_normal(32) * 0.1).astype(np.float32)
    idx, w = oracle.route(logits, bias, 4, "sigmoid", renorm=False)
    s = 1 / (1 + np.exp(-logits.astype(np.float64)))
    assert np.allclose(w, np.take_along_axis(s, idx, 1), rtol=1e-6)


# ---------------------------------------------------------------------------- dispatch
def test_dispatch_invariants():
    rng = np.random.default_rng(8)
    T, E, k = 300, 37, 5
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm_src, slot_of = oracle.dispatch(idx, E)
    S = T * k
    assert counts.sum() == S and offsets[-1] == S and offsets[0] == 0
    assert np.all(np.diff(offsets) >= 0) and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(np.sort(perm_src), np.arange(S))              # bijection
    assert np.array_equal(slot_of[perm_src], np.arange(S))
    flat = idx.reshape(-1)
    for e in range(E):
        src = perm_src[offsets[e]:offsets[e + 1]]
        assert np.all(flat[src] == e)
        assert np.all(np.diff(src // k) > 0)                            # ascending tokens


def test_dispatch_degenerate():
    # every token on one expert, other experts empty
    idx = np.full((10, 1), 3, np.int32)
    counts, offsets, perm_src, slot_of = oracle.dispatch(idx, 5)
    assert list(counts) == [0, 0, 0, 10, 0]
    assert list(offsets) == [0, 0, 0, 0, 10, 10]
    assert np.array_equal(perm_src, np.arange(10))


@pytest.mark.parametrize("act", ["f32", "bf16"])
def test_combine_inverts_dispatch(act):
    rng = np.random.default_rng(9)
    T, E, k, H = 50, 9, 3, 24
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    x = rng.standard_normal((T, H))
    x = x.astype(np.float32).astype(np.float64) if act == "f32" else oracle.round_bf16(x)
    _, _, perm_src, slot_of = oracle.dispatch(idx, E)
    y = x[perm_src // k]                                      # y := x_perm
    w = np.zeros((T, k), np.float32)
    w[:, 0] = 1.0
    assert np.array_equal(oracle.combine(y, slot_of, w, act), x)


# ---------------------------------------------------------------------------- FFN
def _dense_ffn_torch(x, w1, w2):
    x, w1, w2 = (torch.from_numpy(np.asarray(a, np.float64)) for a in (x, w1, w2))
    I = w1.shape[0] // 2
    g = torch.einsum("th,ih->ti", x, w1[:I])
    u = torch.einsum("th,ih->ti", x, w1[I:])
    return torch.einsum("ti,hi->th", torch.nn.functional.silu(g) * u, w2).numpy()


def test_identical_experts_reduce_to_dense_ffn():
    wl = synth.WORKLOADS["tiny_f32"].scaled(T=32, E=6, k=3)
    L = _layer(wl)
    L.w1[:] = L.w1[0]
    L.w2[:] = L.w2[0]
    out = oracle.forward(L)
    ref = _dense_ffn_torch(L.x, L.w1[0], L.w2[0])
    # h and y are stored in fp32 and the gates in fp32: allow a few fp32 roundings
    assert np.max(np.abs(out - ref)) / np.sqrt(np.mean(ref ** 2)) < 2e-6


def test_single_expert_is_dense_ffn():
    wl = synth.WORKLOADS["tiny_f32"].scaled(T=16, E=1, k=1)
    L = _layer(wl)
    r = oracle.forward(L, return_all=True)
    assert np.all(r["topk_w"] == 1.0)
    ref = _dense_ffn_torch(L.x, L.w1[0], L.w2[0])
    assert np.allclose(r["out"], ref, rtol=1e-6, atol=1e-7)


def test_quant_e4m3_block_scale_rule():
    rng = np.random.default_rng(10)
    h = (rng.standard_normal((8, 512)) * np.array([1e-3, 1, 50, 1e4])[:, None].repeat(2, 0)
         ).astype(np.float32)
    h[0, :128] = 0.0                                           # all-zero block
    codes, scales = oracle.quant_e4m3_1x128(h)
    assert scales[0, 0] == 1.0 and np.all(codes[0, :128] == 0)
    blocks = np.abs(h.astype(np.float64)).reshape(8, 4, 128).max(2)
    nz = blocks > 0
    # the scale is the smallest power of two that brings amax within 448
    assert np.all(blocks[nz] <= 448 * scales[nz])
    assert np.all(blocks[nz] > 224 * scales[nz])
    assert np.all(np.log2(scales) == np.round(np.log2(scales)))
    # per element: torch's float8 cast of h / scale gives the same value
    ref = torch.from_numpy((h.reshape(8, 4, 128) / scales[:, :, None]).reshape(8, 512)
                           .astype(np.float32)).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(ref, oracle.e4m3_decode(codes))


# ---------------------------------------------------------------------------- brute force
_E2M1 = [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def _bf_dequant_w(w, s, wt, r, c):
    if wt == "f32":
        return float(w[r, c])
    if wt == "bf16":
        return float(np.array([int(w[r, c]) << 16], np.uint32).view(np.float32)[0])
    if wt == "e4m3":
        v = float(torch.tensor([w[r, c]], dtype=torch.uint8).view(torch.float8_e4m3fn)
                  .double())
        return v * float(s[r // 128, c // 128])
    b = int(w[r, c // 2])
    code = (b >> 4) if c % 2 else (b & 15)
    v = _E2M1[code & 7] * (-1 if code & 8 else 1)
    return v * 2.0 ** (int(s[r, c // 32]) - 127)


def _bf_store(v, fmt):
    """Storage rounding by torch's casts (fp64 -> fp32 [-> bf16])."""
    t = torch.tensor([v], dtype=torch.float64).float()
    return float(t) if fmt == "f32" else float(t.to(torch.bfloat16).double())


def _bf_quant_block(vals):
    """E4M3 1x128 contract rounding of one block by scalar loops and torch's cast."""
    v32 = [float(np.float32(a)) for a in vals]
    amax = max(abs(a) for a in v32)
    if amax == 0:
        return [0.0] * len(v32)
    n = 0
    while amax > 448 * 2.0 ** n:
        n += 1
    while amax <= 448 * 2.0 ** (n - 1):
        n -= 1
    s = 2.0 ** n
    q = torch.tensor([a / s for a in v32], dtype=torch.float32).to(torch.float8_e4m3fn)
    return [float(c) * s for c in q.double()]


def _brute_force_layer(L):
    T, E, k = L.T, L.E, L.k
    H = L.w1.shape[2] * (2 if L.wt == "e2m1" else 1)
    I = L.w2.shape[2] * (2 if L.wt == "e2m1" else 1)
    if L.score == "softmax":
        keys = L.logits
    else:
        keys = (oracle.sigmoid_f32(L.logits) + (L.bias if L.bias is not None else 0)
                ).astype(np.float32)
    out = np.zeros((T, H))
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(keys[t, e]), e))[:k]
        if L.score == "softmax":
            z = [math.exp(float(L.logits[t, e]) - float(L.logits[t, order[0]])) for e in order]
        else:
            z = [float(oracle.sigmoid_f32(L.logits[t:t + 1, e])[0]) for e in order]
        gates = [float(np.float32(a / sum(z))) for a in z]
        if L.act == "f32":
            xt = [float(a) for a in L.x[t]]
        elif L.act == "bf16":
            xt = [float(np.array([int(b) << 16], np.uint32).view(np.float32)[0])
                  for b in L.x[t]]
        else:
            xt = [float(torch.tensor([b], dtype=torch.uint8).view(torch.float8_e4m3fn)
                        .double()) * float(L.x_scales[t, c // 128])
                  for c, b in enumerate(L.x[t])]
        acc = [0.0] * H
        for j, e in enumerate(order):
            s1 = None if L.w1_scales is None else L.w1_scales[e]
            s2 = None if L.w2_scales is None else L.w2_scales[e]
            h = []
            for i in range(I):
                g = sum(xt[c] * _bf_dequant_w(L.w1[e], s1, L.wt, i, c) for c in range(H))
                u = sum(xt[c] * _bf_dequant_w(L.w1[e], s1, L.wt, I + i, c) for c in range(H))
                h.append(g / (1 + math.exp(-g)) * u)
            if L.act == "e4m3":
                hq = []
                for b0 in range(0, I, 128):
                    hq += _bf_quant_block(h[b0:b0 + 128])
                h = hq
            else:
                h = [_bf_store(a, L.act) for a in h]
            for c in range(H):
                y = sum(h[i] * _bf_dequant_w(L.w2[e], s2, L.wt, c, i) for i in range(I))
                acc[c] += gates[j] * _bf_store(y, "f32" if L.act == "f32" else "bf16")
        out[t] = [_bf_store(a, "f32" if L.act == "f32" else "bf16") for a in acc]
    return out


@pytest.mark.parametrize("act,wt,score", [("f32", "f32", "softmax"),
                                          ("bf16", "bf16", "softmax"),
                                          ("e4m3", "e4m3", "sigmoid"),
                                          ("e4m3", "e2m1", "softmax")])
def test_layer_brute_force(act, wt, score):
    H, I = (128, 128)
    wl = synth.Workload("bf", 3, H, 4, 2, I, act, wt, score, "normal", bias=score == "sigmoid")
    L = _layer(wl)
    got = oracle.forward(L)
    ref = _brute_force_layer(L)
    scale = np.sqrt(np.mean(ref ** 2))
    # the brute force sums in a different order; outputs are stored in bf16 / fp32, so at
    # most one storage ulp apart
    tol = 1e-6 if act == "f32" else 2 ** -7
    assert np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * scale)) <= tol


def test_forward_tokens_and_slots_agree_with_forward():
    wl = synth.WORKLOADS["v3_fp8"].scaled(T=40, H=256, E=8, k=3, I=256)
    L = _layer(wl)
    r = oracle.forward(L, return_all=True)
    toks = np.array([0, 7, 39, 12])
    assert np.array_equal(oracle.forward_tokens(L, toks), r["out"][toks])
    slots = np.array([0, 5, 60, 119])
    assert np.array_equal(oracle.ffn_slots(L, slots, r["perm_src"], r["offsets"]),
                          r["y"][slots])


def test_synth_e4m3_decodes_like_torch():
    wl = synth.WORKLOADS["v3_fp8"].scaled(T=4, H=256, E=2, k=1, I=128)
    d = synth.make_inputs(wl)
    ref = d["x"].view(torch.float8_e4m3fn).double() * d["x_scales"].double() \
        .repeat_interleave(128, 1)
    got = oracle.dequant_x(d["x"].numpy(), d["x_scales"].numpy(), "e4m3")
    assert np.array_equal(ref.numpy(), got)


# ----------------------------------------------------------------------- group-limited routing
def _route_grouped_brute(keys, k, n_group, topk_group):
    """Plain-Python restatement: group score = sum of a group's two largest keys (fp32 add),
    keep the topk_group best groups (ties -> lower group), then the k best experts of the
    kept groups (ties -> lower expert)."""
    T, E = keys.shape
    G = E // n_group
    out = []
    for t in range(T):
        gs = []
        for g in range(n_group):
            ks = sorted((float(keys[t, e]) for e in range(g * G, (g + 1) * G)), reverse=True)
            sc = ks[0] if G == 1 else float(np.float32(ks[0]) + np.float32(ks[1]))
            gs.append((-sc, g))
        kept = {g for _, g in sorted(gs)[:topk_group]}
        cand = sorted((-float(keys[t, e]), e) for e in range(E) if e // G in kept)
        out.append([e for _, e in cand[:k]])
    return np.array(out, np.int32)


@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
@pytest.mark.parametrize("E,n_group,topk_group,k", [(16, 4, 2, 3), (32, 8, 3, 4), (12, 12, 5, 5),
                                                    (64, 2, 1, 8)])
def test_route_grouped_brute_force(score, E, n_group, topk_group, k):
    rng = np.random.default_rng(E + n_group)
    logits = rng.standard_normal((40, E)).astype(np.float32)
    logits[::5] = np.round(logits[::5])            # many equal keys and group scores
    bias = (rng.standard_normal(E) * 0.1).astype(np.float32)
    idx, _ = oracle.route(logits, bias if score == "sigmoid" else None, k, score,
                          n_group=n_group, topk_group=topk_group)
    keys = logits if score == "softmax" else (oracle.sigmoid_f32(logits) + bias).astype(np.float32)
    assert np.array_equal(idx, _route_grouped_brute(keys, k, n_group, topk_group))


def test_route_grouped_all_groups_is_plain_routing_and_scale_multiplies():
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((20, 64)).astype(np.float32)
    bias = (rng.standard_normal(64) * 0.1).astype(np.float32)
    for score in ("softmax", "sigmoid"):
        b = bias if score == "sigmoid" else None
        i0, w0 = oracle.route(logits, b, 6, score)
        i1, w1 = oracle.route(logits, b, 6, score, n_group=8, topk_group=8, scale=2.5)
        assert np.array_equal(i0, i1)
        assert np.array_equal(w0 * 2.5, w1)


def test_route_grouped_excludes_a_strong_expert_in_a_weak_group():
    # group 0 holds the single best expert but a weak second; groups 1 and 2 are stronger
    # by their top-2 sums, so with topk_group = 2 expert 0 must not be chosen
    keys = np.array([[5.0, -9, -9, -9, 3, 3, -9, -9, 2.9, 2.9, -9, -9]], np.float32)
    idx, _ = oracle.route(keys, None, 2, "softmax", n_group=3, topk_group=2)
    assert idx.tolist() == [[4, 5]]


def test_dequant_takes_any_fp32_block_scale():
    """The oracle's dequantisation is code x block scale for any fp32 scale, not only powers of
    two (the GPU path refuses other scales; the definition does not depend on them)."""
    rng = np.random.default_rng(12)
    w = rng.integers(0, 256, (256, 384), dtype=np.uint8)
    w[(w & 0x7F) == 0x7F] = 0                                  # no NaN codes
    s = rng.uniform(0.1, 3.0, (2, 3)).astype(np.float32)       # non-power-of-two scales
    d = oracle.dequant_w(w, s, "e4m3")
    for _ in range(200):
        r, c = int(rng.integers(0, 256)), int(rng.integers(0, 384))
        assert d[r, c] == _bf_dequant_w(w, s, "e4m3", r, c)
    x = rng.integers(0, 256, (5, 256), dtype=np.uint8)
    x[(x & 0x7F) == 0x7F] = 0
    xs = rng.uniform(0.1, 3.0, (5, 2)).astype(np.float32)
    dx = oracle.dequant_x(x, xs, "e4m3")
    ref = torch.from_numpy(x).view(torch.float8_e4m3fn).double().numpy() * \
        np.repeat(xs.astype(np.float64), 128, axis=1)
    assert np.array_equal(dx, ref)
