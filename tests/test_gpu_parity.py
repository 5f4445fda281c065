"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integer results (routing indices, counts, offsets, permutations, dispatched bytes) must match
bit for bit.  Floating-point outputs must satisfy max|gpu - oracle| / rms(oracle) <= 1e-4
(fp32 layer), 1e-2 (BF16) or 3e-2 (FP8 / FP4).  Sizes are chosen so that the oracle finishes
in seconds while the GEMMs still span several tiles with ragged tails; the full-size
workloads are checked on sampled tokens."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.util import (TOL, assert_parity, assert_within_bound, combine_allowance,
                        fp32_sum_bound, host_values,
                        oracle_layer, parity_err, raw_err, weights_of)

pytestmark = pytest.mark.gpu

M = pytest.importorskip("moe_expert_layer_prefix_b200")
DEV = "cuda"

SMALL = {
    "tiny_f32": synth.WORKLOADS["tiny_f32"],
    "mixtral_bf16": synth.WORKLOADS["mixtral_bf16"].scaled(T=200, H=512, I=1024),
    "mixtral_bf16_h384": synth.WORKLOADS["mixtral_bf16"].scaled(T=77, H=384, E=5, I=256),
    "v3_fp8": synth.WORKLOADS["v3_fp8"].scaled(T=300, H=1024, E=16, k=4, I=512),
    "decode_fp8_fp4": synth.WORKLOADS["decode_fp8_fp4"].scaled(T=33, H=1024, E=64, I=256),
    "skewed_fp8_fp4": synth.WORKLOADS["skewed_fp8_fp4"].scaled(T=260, H=512, E=128, I=256),
    # at least 128 rows per expert on average: 2-CTA (M = 256) tiles
    "v3_fp8_pair": synth.WORKLOADS["v3_fp8"].scaled(T=600, H=1024, E=8, k=4, I=512),
    "mixtral_bf16_pair": synth.WORKLOADS["mixtral_bf16"].scaled(T=512, H=512, E=4, I=512),
    "mixtral_bf16_h384_pair": synth.WORKLOADS["mixtral_bf16"].scaled(T=400, H=384, E=3, I=256),
    "skewed_fp8_fp4_pair": synth.WORKLOADS["skewed_fp8_fp4"].scaled(T=512, H=512, E=32, k=8,
                                                                    I=256),
    # 32-row tiles forced on shapes that would not pick them (several m-blocks per expert)
    "v3_fp8_small": synth.WORKLOADS["v3_fp8"].scaled(T=300, H=1024, E=16, k=4, I=512),
    "skewed_fp8_fp4_small": synth.WORKLOADS["skewed_fp8_fp4"].scaled(T=260, H=512, E=128,
                                                                     I=256),
    "mixtral_bf16_h384_small": synth.WORKLOADS["mixtral_bf16"].scaled(T=77, H=384, E=5, I=256),
}


@pytest.fixture(autouse=True)
def _clear_device_error(request):
    """Each test starts with a clear device error word (and asserts on its own errors);
    configurations named *_small run with 32-row tiles forced."""
    M.moe_get_device_error()
    name = getattr(request.node, "callspec", None)
    small = name is not None and str(name.params.get("name", "")).endswith("_small")
    if small:
        M.moe_set_gemm_tiles("small")
    try:
        yield
    finally:
        if small:
            M.moe_set_gemm_tiles("auto")


def _inputs(wl):
    return synth.make_inputs(wl, DEV)


# ------------------------------------------------------------------------------- route
@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_route_full_size_bit_exact(name):
    wl = synth.WORKLOADS[name]
    a = synth.make_activations(wl, DEV)
    idx, w = M.moe_route(a["logits"], wl.k, wl.score, bias=a["bias"], renorm=wl.renorm)
    ridx, rw = oracle.route(a["logits"].cpu().numpy(),
                            None if a["bias"] is None else a["bias"].cpu().numpy(), wl.k,
                            wl.score, wl.renorm)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.max(np.abs(w.cpu().numpy() - rw) / rw) < 1e-6


@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
@pytest.mark.parametrize("T,E,k", [(1, 8, 1), (5, 8, 8), (37, 1024, 32), (64, 33, 3), (9, 1, 1)])
def test_route_edges(score, T, E, k):
    g = torch.Generator(device=DEV).manual_seed(T * 131 + E)
    logits = torch.randn((T, E), generator=g, device=DEV)
    logits[0] = 0.5                                         # all tied
    bias = torch.randn(E, generator=g, device=DEV) * 0.1 if score == "sigmoid" else None
    for renorm in (True, False):
        idx, w = M.moe_route(logits, k, score, bias=bias, renorm=renorm)
        ridx, rw = oracle.route(logits.cpu().numpy(),
                                None if bias is None else bias.cpu().numpy(), k, score, renorm)
        assert np.array_equal(idx.cpu().numpy(), ridx)
        assert np.max(np.abs(w.cpu().numpy() - rw) / np.maximum(rw, 1e-30)) < 2e-6


@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
@pytest.mark.parametrize("E,k", [(256, 8), (1024, 16), (1024, 32), (100, 5)])
def test_route_tied_keys(score, E, k):
    """Keys that tie at and around the k-th best: logits on a coarse grid (a few dozen to
    hundreds of equal keys per row), +0 / -0 mixes and -inf logits.  The router's selection
    takes its exact candidate ranking when few keys reach its bound and its fallback when
    many do; both must give the oracle's (key desc, id asc) order."""
    g = torch.Generator(device=DEV).manual_seed(E * 7 + k)
    T = 96
    logits = torch.round(torch.randn((T, E), generator=g, device=DEV) * 2.0) / 2.0
    logits[1::3] = torch.round(torch.randn((T // 3, E), generator=g, device=DEV) * 0.3)
    zeros = torch.zeros(E, device=DEV)
    zeros[torch.arange(0, E, 2, device=DEV)] = -0.0
    logits[2] = zeros                                         # +0 / -0 only
    logits[5, torch.arange(0, E, 3, device=DEV)] = float("-inf")
    bias = torch.randn(E, generator=g, device=DEV) * 0.1 if score == "sigmoid" else None
    for renorm in (True, False):
        idx, w = M.moe_route(logits, k, score, bias=bias, renorm=renorm)
        ridx, rw = oracle.route(logits.cpu().numpy(),
                                None if bias is None else bias.cpu().numpy(), k, score, renorm)
        assert np.array_equal(idx.cpu().numpy(), ridx)
        assert np.max(np.abs(w.cpu().numpy() - rw) / np.maximum(rw, 1e-30)) < 2e-6


# ------------------------------------------------------------------------------- dispatch
def _check_dispatch(wl, d, idx):
    r = M.moe_dispatch(d["x"], idx, wl.E, wl.act, x_scales=d["x_scales"])
    counts, offs, perm_src, slot_of = oracle.dispatch(idx.cpu().numpy(), wl.E)
    assert np.array_equal(r["expert_offsets"].cpu().numpy(), offs)
    assert np.array_equal(r["perm_src"].cpu().numpy(), perm_src)
    assert np.array_equal(r["slot_of"].cpu().numpy(), slot_of)
    tok = torch.from_numpy(perm_src // wl.k).long().to(DEV)
    assert torch.equal(r["x_perm"], d["x"][tok])
    if wl.act == "e4m3":
        assert torch.equal(r["x_perm_scales"], d["x_scales"][tok])
    return r


@pytest.mark.parametrize("name", list(SMALL))
def test_dispatch_bit_exact(name):
    wl = SMALL[name]
    d = _inputs(wl)
    idx, _ = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"])
    _check_dispatch(wl, d, idx)


@pytest.mark.parametrize("case", ["one_expert", "empty_experts", "T1"])
def test_dispatch_edges(case):
    wl = synth.WORKLOADS["v3_fp8"].scaled(T=70, H=256, E=40, k=3, I=128)
    if case == "T1":
        wl = wl.scaled(T=1)
    d = _inputs(wl)
    if case == "one_expert":
        idx = torch.tensor([[7, 3, 9]] * wl.T, dtype=torch.int32, device=DEV)
    elif case == "empty_experts":
        idx = torch.stack([torch.randperm(5, device=DEV)[:3] for _ in range(wl.T)]).int() + 30
    else:
        idx = torch.tensor([[39, 0, 12]], dtype=torch.int32, device=DEV)
    _check_dispatch(wl, d, idx)


def test_dispatch_full_size_bit_exact():
    wl = synth.WORKLOADS["skewed_fp8_fp4"]
    a = synth.make_activations(wl, DEV)
    idx, _ = M.moe_route(a["logits"], wl.k, wl.score)
    _check_dispatch(wl, a, idx)


# ------------------------------------------------------------------------------- combine
@pytest.mark.parametrize("ydt", ["bf16", "f32"])
def test_combine(ydt):
    T, k, H, E = 123, 5, 768, 20
    g = torch.Generator(device=DEV).manual_seed(5)
    logits = torch.randn((T, E), generator=g, device=DEV)
    idx, w = M.moe_route(logits, k)
    d = M.moe_dispatch(torch.randn((T, H), device=DEV), idx, E, "f32")
    y = torch.randn((T * k, H), generator=g, device=DEV)
    y = y if ydt == "f32" else y.to(torch.bfloat16)
    out = M.moe_combine(y, d["slot_of"], w)
    ref = oracle.combine(host_values(y, None, ydt), d["slot_of"].cpu().numpy(),
                         w.cpu().numpy(), ydt)
    got = host_values(out, None, ydt)
    assert_parity(got, ref, ydt, 1e-6 if ydt == "f32" else 1e-3)


def test_combine_inverts_dispatch():
    T, k, H, E = 50, 3, 256, 9
    x = torch.randn((T, H), device=DEV).to(torch.bfloat16)
    idx, _ = M.moe_route(torch.randn((T, E), device=DEV), k)
    d = M.moe_dispatch(x, idx, E, "bf16")
    w = torch.zeros((T, k), device=DEV)
    w[:, 0] = 1.0
    assert torch.equal(M.moe_combine(d["x_perm"], d["slot_of"], w), x)


# ------------------------------------------------------------------------------- expert FFN
def _expert_ffn_ref(L, wl, xh_rows_by_expert, offsets):
    """oracle y and stored h, expert by expert, on given dequantised input rows."""
    S = offsets[-1]
    y = np.zeros((S, wl.H))
    h = np.zeros((S, wl.I))
    for e in range(wl.E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        w1, w2 = L.expert_weights(e)
        y[a:b], h[a:b] = oracle.expert_ffn(xh_rows_by_expert[a:b], w1, w2, wl.act,
                                           return_h=True)
    return y, h


@pytest.mark.parametrize("name", list(SMALL))
def test_linear1_linear2(name):
    wl = SMALL[name]
    d = _inputs(wl)
    W = weights_of(wl, d)
    idx, _ = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"])
    r = M.moe_dispatch(d["x"], idx, wl.E, wl.act, x_scales=d["x_scales"])
    h, hs = M.moe_expert_linear1(r["x_perm"], r["expert_offsets"], W,
                                 x_perm_scales=r["x_perm_scales"])
    y = M.moe_expert_linear2(h, r["expert_offsets"], W, h_scales=hs)
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    L = oracle_layer(wl, d)
    offs = r["expert_offsets"].cpu().numpy()
    xp = host_values(r["x_perm"], r["x_perm_scales"], wl.act)
    yref, href = _expert_ffn_ref(L, wl, xp, offs)
    hg = host_values(h, hs, wl.act)
    if wl.act == "e4m3":
        # h codes: the GPU decides on its fp32 h, the oracle on its fp64 h rounded to fp32,
        # so a code may land one E4M3 step away (a block scale two-fold away when amax sits
        # on a power-of-two boundary); everything else must be identical
        sub = np.repeat(np.maximum(hs.cpu().numpy(), 1e-30).astype(np.float64), 128, 1)
        dh = np.abs(hg - href)
        assert np.all((dh <= 0.126 * np.abs(href) + 1e-30) | (dh <= 2 * 2 ** -9 * sub))
        assert np.mean(hg != href) < 0.01
    else:
        # BF16 / fp32 h: the GPU sums gate and up in fp32 over K = H products (exact in
        # fp32), so each is within fp32_sum_bound of the exact value; h = silu(g) * u
        # carries that error through |dh/dg| = |u| |silu'(g)| <= 1.1 |u| and
        # |dh/du| = |silu(g)|, plus the fast exponential and division of the epilogue
        # (relative error below (|g| + 8) * 2^-22); then both sides round to the storage
        # format
        bnd = np.zeros_like(href)
        for e in range(wl.E):
            a, b = int(offs[e]), int(offs[e + 1])
            if a == b:
                continue
            w1, _ = L.expert_weights(e)
            xa = np.abs(xp[a:b])
            g = xp[a:b] @ w1[:wl.I].T
            u = xp[a:b] @ w1[wl.I:].T
            bg = fp32_sum_bound(xa @ np.abs(w1[:wl.I]).T, wl.H)
            bu = fp32_sum_bound(xa @ np.abs(w1[wl.I:]).T, wl.H)
            with np.errstate(over="ignore"):
                silu = g / (1.0 + np.exp(-g))
            bnd[a:b] = (1.1 * (np.abs(u) + bu) * bg + (np.abs(silu) + 1.1 * bg) * bu +
                        (np.abs(g) + 8) * 2.0 ** -22 * np.abs(silu * u))
        assert_within_bound(hg, href, bnd, wl.act, "h")
    # y: linear-2 alone, on the GPU's own h (only accumulation order and the output
    # rounding differ): within the fp32 accumulation bound over K = I, then rounded
    y2ref = np.zeros_like(yref)
    y2bnd = np.zeros_like(yref)
    for e in range(wl.E):
        a, b = int(offs[e]), int(offs[e + 1])
        if a < b:
            _, w2 = L.expert_weights(e)
            y2ref[a:b] = hg[a:b] @ w2.T
            y2bnd[a:b] = fp32_sum_bound(np.abs(hg[a:b]) @ np.abs(w2).T, wl.I)
    yfmt = "f32" if wl.act == "f32" else "bf16"
    yg = host_values(y, None, yfmt)
    assert_within_bound(yg, y2ref, y2bnd, yfmt, "y on the GPU's h")
    # y against the oracle's own h
    assert_parity(yg, yref, yfmt, TOL[wl.act])


# ------------------------------------------------------------------------------- forward
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_end_to_end(name):
    wl = SMALL[name]
    d = _inputs(wl)
    W = weights_of(wl, d)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device=DEV)
    out = M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, bias=d["bias"],
                        renorm=wl.renorm, x_scales=d["x_scales"], topk_idx=idx)
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    L = oracle_layer(wl, d)
    r = oracle.forward(L, return_all=True)
    assert np.array_equal(idx.cpu().numpy(), r["topk_idx"])
    fmt = "f32" if wl.act == "f32" else "bf16"
    allow = combine_allowance(r["y"][r["slot_of"].reshape(wl.T, wl.k)],
                              r["topk_w"].astype(np.float32), fmt)
    mx, l2, raw = assert_parity(host_values(out, None, fmt), r["out"], fmt, TOL[wl.act],
                                allow=allow)
    print(f"\n[parity] {name}: raw max|gpu-oracle|/rms(oracle) = {raw:.3e}, "
          f"max-excess/rms = {mx:.3e}, rel-L2 = {l2:.3e}, tol = {TOL[wl.act]}")


@pytest.mark.parametrize("name", ["v3_fp8", "skewed_fp8_fp4", "mixtral_bf16",
                                  "v3_fp8_pair", "skewed_fp8_fp4_pair", "decode_fp8_fp4",
                                  "v3_fp8_small"])
def test_forward_equals_unfused_chain(name):
    """moe_forward (one persistent launch) produces exactly the bytes of the chain of entry
    points (same device code, same tile order; the same single-CTA tile shape for both)."""
    wl = SMALL[name]
    d = _inputs(wl)
    W = weights_of(wl, d)
    M.moe_set_gemm_tiles("small" if name.endswith("_small") or name.startswith("decode")
                         else "single")
    try:
        idx1 = torch.empty((wl.T, wl.k), dtype=torch.int32, device=DEV)
        out = M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, bias=d["bias"],
                            x_scales=d["x_scales"], topk_idx=idx1)
        idx, w = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"])
        r = M.moe_dispatch(d["x"], idx, wl.E, wl.act, x_scales=d["x_scales"])
        y = M.moe_fused_ffn(r["x_perm"], r["expert_offsets"], W,
                            x_perm_scales=r["x_perm_scales"])
        out2 = M.moe_combine(y, r["slot_of"], w)
        torch.cuda.synchronize()
        assert M.moe_get_device_error()[0] == 0
    finally:
        M.moe_set_gemm_tiles("auto")
    assert torch.equal(idx1, idx)
    assert torch.equal(out, out2)


@pytest.mark.parametrize("name", ["v3_fp8", "skewed_fp8_fp4", "mixtral_bf16_h384"])
def test_small_tiles_equal_single(name):
    """32-row and 128-row tiles run the same M = 128 MMAs over the same K order on each
    row, so the expert GEMMs give the same bits either way."""
    wl = SMALL[name]
    d = _inputs(wl)
    W = weights_of(wl, d)
    idx, _ = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"])
    r = M.moe_dispatch(d["x"], idx, wl.E, wl.act, x_scales=d["x_scales"])
    res = []
    try:
        for mode in ("single", "small"):
            M.moe_set_gemm_tiles(mode)
            h, hs = M.moe_expert_linear1(r["x_perm"], r["expert_offsets"], W,
                                         x_perm_scales=r["x_perm_scales"])
            y = M.moe_expert_linear2(h, r["expert_offsets"], W, h_scales=hs)
            torch.cuda.synchronize()
            assert M.moe_get_device_error()[0] == 0
            res.append((h, hs, y))
    finally:
        M.moe_set_gemm_tiles("auto")
    (h1, hs1, y1), (h2, hs2, y2) = res
    assert torch.equal(h1, h2)
    assert hs1 is None or torch.equal(hs1, hs2)
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("wl", [
    synth.WORKLOADS["v3_fp8"].scaled(T=3000, H=512, E=16, k=4, I=256),
    synth.WORKLOADS["mixtral_bf16"].scaled(T=2500, H=384, E=5, I=256),
    synth.WORKLOADS["skewed_fp8_fp4"].scaled(T=2400, H=768, E=64, k=16, I=256),
], ids=["v3_fp8", "mixtral_bf16_h384", "skewed_fp8_fp4"])
def test_forward_many_tokens_equals_unfused_chain(wl):
    """Enough tokens (T >= 2 x the persistent kernel's warps) for its whole-row combine
    path: still the chain's bytes."""
    d = _inputs(wl)
    W = weights_of(wl, d)
    M.moe_set_gemm_tiles("single")
    try:
        out = M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, bias=d["bias"],
                            x_scales=d["x_scales"])
        idx, w = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"])
        r = M.moe_dispatch(d["x"], idx, wl.E, wl.act, x_scales=d["x_scales"])
        y = M.moe_fused_ffn(r["x_perm"], r["expert_offsets"], W,
                            x_perm_scales=r["x_perm_scales"])
        out2 = M.moe_combine(y, r["slot_of"], w)
        torch.cuda.synchronize()
        assert M.moe_get_device_error()[0] == 0
    finally:
        M.moe_set_gemm_tiles("auto")
    assert torch.equal(out, out2)


def test_forward_deterministic():
    wl = SMALL["skewed_fp8_fp4"]
    d = _inputs(wl)
    W = weights_of(wl, d)
    a = M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, x_scales=d["x_scales"])
    b = M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, x_scales=d["x_scales"])
    assert M.moe_get_device_error()[0] == 0
    assert torch.equal(a, b)


def _sample_tokens(offsets, perm_src, k, T, n=32, seed=0):
    """At least n tokens of a full-size layer, chosen to reach the tiles most likely to go
    wrong: rows of the most-loaded expert (first, last, m-block boundaries), the tokens of
    experts with a single row (or the fewest rows), the last row of every expert whose count
    leaves a ragged 128-row m-block (up to 8 of them, the last touched expert first), then
    random tokens."""
    counts = np.diff(offsets)
    tok_of = lambda slot: int(perm_src[slot]) // k  # noqa: E731
    pick = []
    e_max = int(np.argmax(counts))
    a, b = int(offsets[e_max]), int(offsets[e_max + 1])
    for slot in (a, a + 127, a + 128, (a + b) // 2, b - 1):
        if a <= slot < b:
            pick.append(tok_of(slot))
    touched = np.nonzero(counts)[0]
    fewest = touched[np.argsort(counts[touched], kind="stable")][:4]
    pick += [tok_of(int(offsets[e])) for e in fewest]
    ragged = [int(e) for e in touched[::-1] if counts[e] % 128][:8]
    pick += [tok_of(int(offsets[e + 1]) - 1) for e in ragged]
    rng = np.random.default_rng(seed)
    seen = []
    for t in pick + list(rng.permutation(T)):
        if t not in seen:
            seen.append(int(t))
        if len(seen) >= max(n, len(set(pick))):
            break
    return np.array(seen, dtype=np.int64)


@pytest.mark.parametrize("name", ["v3_fp8", "decode_fp8_fp4", "mixtral_bf16", "skewed_fp8_fp4"])
def test_forward_full_size_sampled(name):
    """The full-size workload in the benchmark's launch configuration: routing and dispatch
    compared for every token, the output on >= 32 tokens chosen to cover the most-loaded
    expert, the smallest experts and ragged m-block tails, normalised by the RMS of the
    oracle's rows."""
    wl = synth.WORKLOADS[name]
    d = _inputs(wl)
    W = weights_of(wl, d)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device=DEV)
    offs_gpu = torch.empty(wl.E + 1, dtype=torch.int32, device=DEV)
    out = M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, bias=d["bias"],
                        x_scales=d["x_scales"], topk_idx=idx, expert_offsets=offs_gpu)
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    L = oracle_layer(wl, d, lazy_weights=True)
    ridx, _ = oracle.route(L.logits, L.bias, wl.k, wl.score, wl.renorm)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    _, roffs, rperm, _ = oracle.dispatch(ridx, wl.E)
    assert np.array_equal(offs_gpu.cpu().numpy(), roffs)
    toks = _sample_tokens(roffs, rperm, wl.k, wl.T)
    assert toks.size >= 32
    ref, y_ref, w_ref = oracle.forward_tokens(L, toks, return_y=True)
    got = host_values(out[torch.from_numpy(toks).to(DEV)], None, "bf16")
    mx, l2, raw = assert_parity(got, ref, "bf16", TOL[wl.act],
                                allow=combine_allowance(y_ref, w_ref, "bf16"))
    print(f"\n[full-size parity] {name}: {toks.size} tokens, raw max|gpu-oracle|/rms(oracle) "
          f"= {raw:.3e}, max-excess/rms = {mx:.3e}, rel-L2 = {l2:.3e}, tol = {TOL[wl.act]}")


# ------------------------------------------------------------------------------- errors
def test_invalid_arguments_rejected_before_launch():
    x = torch.zeros((4, 128), device=DEV)
    with pytest.raises(M.MoeError) as ei:
        M.moe_route(torch.zeros((4, 2000), device=DEV), 2)
    assert ei.value.status == -2
    with pytest.raises(M.MoeError) as ei:
        M.moe_route(torch.zeros((4, 8), device=DEV), 9)
    assert ei.value.status == -2
    idx = torch.zeros((4, 1), dtype=torch.int32, device=DEV)
    with pytest.raises(M.MoeError) as ei:
        M.moe_dispatch(x, idx, 8, "f32", ws=torch.empty(1, dtype=torch.uint8, device=DEV))
    assert ei.value.status == -4
