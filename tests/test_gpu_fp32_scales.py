"""Arbitrary (non-power-of-two) fp32 block scales on the E4M3 layer, through the C ABI.

The layer's scales are fp32 per 1x128 activation block and per 128x128 weight block (youleyou,
"DeepSeek 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", section "Tile Kernels：逼近硬件极限的底层
优化", quantisation item).  With scale_fmt 'fp32' the expert GEMMs fold every 128-deep block's
partial sum into an fp32 accumulator with its scales; the oracle dequantises code x scale
element by element in fp64 and is unchanged.  Inputs: the synthetic power-of-two scales
multiplied by seeded factors in [1.05, 1.95], so that no scale is a power of two."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.util import (TOL, assert_parity, assert_within_bound, combine_allowance, fp32_sum_bound,
                        host_values, oracle_layer)

pytestmark = pytest.mark.gpu

M = pytest.importorskip("moe_expert_layer_prefix_b200")
DEV = "cuda"

CASES = {
    "v3_fp8": synth.WORKLOADS["v3_fp8"].scaled(T=300, H=1024, E=16, k=4, I=512),
    # K = 384 (three 128-blocks, rows not 16-byte aligned in the scale arrays), I = 256
    "v3_fp8_h384": synth.WORKLOADS["v3_fp8"].scaled(T=130, H=384, E=5, k=2, I=256),
    # several m-blocks per expert and a ragged last one
    "v3_fp8_many_rows": synth.WORKLOADS["v3_fp8"].scaled(T=700, H=512, E=4, k=2, I=384),
}


def _fp32_scaled_inputs(wl, seed=0):
    d = synth.make_inputs(wl, DEV)
    g = torch.Generator(device=DEV).manual_seed(1234 + seed)
    for name in ("x_scales", "w1_scales", "w2_scales"):
        f = 1.05 + 0.9 * torch.rand(d[name].shape, generator=g, device=DEV)
        d[name] = (d[name] * f).contiguous()
    for name in ("x_scales", "w1_scales", "w2_scales"):
        m = torch.frexp(d[name].cpu())[0]
        assert not bool((m == 0.5).any()), name   # no scale is a power of two
    return d


def _weights(wl, d):
    return M.Weights(wl.act, wl.wt, d["w1"], d["w2"], d["w1_scales"], d["w2_scales"],
                     scale_fmt="fp32")


@pytest.mark.parametrize("name", list(CASES))
def test_fp32_scales_chain_matches_oracle(name):
    wl = CASES[name]
    d = _fp32_scaled_inputs(wl)
    W = _weights(wl, d)
    idx, w = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"])
    r = M.moe_dispatch(d["x"], idx, wl.E, wl.act, x_scales=d["x_scales"])
    h, hs = M.moe_expert_linear1(r["x_perm"], r["expert_offsets"], W,
                                 x_perm_scales=r["x_perm_scales"])
    y = M.moe_expert_linear2(h, r["expert_offsets"], W, h_scales=hs)
    out = M.moe_combine(y, r["slot_of"], w)
    torch.cuda.synchronize()
    st, site = M.moe_get_device_error()
    assert st == 0, (st, site)
    L = oracle_layer(wl, d)
    offs = r["expert_offsets"].cpu().numpy()
    xp = host_values(r["x_perm"], r["x_perm_scales"], wl.act)
    # h: E4M3 codes within one step of the oracle's on the same (dequantised) rows
    href = np.zeros((wl.S, wl.I))
    for e in range(wl.E):
        a, b = int(offs[e]), int(offs[e + 1])
        if a < b:
            w1, w2 = L.expert_weights(e)
            _, href[a:b] = oracle.expert_ffn(xp[a:b], w1, w2, wl.act, return_h=True)
    hg = host_values(h, hs, wl.act)
    sub = np.repeat(np.maximum(hs.cpu().numpy(), 1e-30).astype(np.float64), 128, 1)
    dh = np.abs(hg - href)
    assert np.all((dh <= 0.126 * np.abs(href) + 1e-30) | (dh <= 2 * 2 ** -9 * sub))
    assert np.mean(hg != href) < 0.01
    # y from the GPU's own h: within the fp32 bound of a blockwise sum (K products, one
    # partial per 128-block scaled once and added once)
    yg = host_values(y, None, "bf16")
    y2 = np.zeros((wl.S, wl.H))
    yb = np.zeros((wl.S, wl.H))
    for e in range(wl.E):
        a, b = int(offs[e]), int(offs[e + 1])
        if a < b:
            _, w2 = L.expert_weights(e)
            y2[a:b] = hg[a:b] @ w2.T
            yb[a:b] = fp32_sum_bound(np.abs(hg[a:b]) @ np.abs(w2).T, wl.I + 3 * (wl.I // 128))
    assert_within_bound(yg, y2, yb, "bf16", "y on the GPU's h")
    # the layer end to end
    ref = oracle.forward(L, return_all=True)
    allow = combine_allowance(ref["y"][ref["slot_of"].reshape(wl.T, wl.k)],
                              ref["topk_w"].astype(np.float32), "bf16")
    mx, l2, raw = assert_parity(host_values(out, None, "bf16"), ref["out"], "bf16", TOL[wl.act],
                                allow=allow)
    print(f"\n[fp32 scales] {name}: raw {raw:.3e} max-excess {mx:.3e} rel-L2 {l2:.3e}")


def test_fp32_scales_forward_equals_chain_and_pow2_path_refuses():
    wl = CASES["v3_fp8"]
    d = _fp32_scaled_inputs(wl, seed=1)
    W = _weights(wl, d)
    out = M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, bias=d["bias"],
                        x_scales=d["x_scales"])
    idx, w = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"])
    r = M.moe_dispatch(d["x"], idx, wl.E, wl.act, x_scales=d["x_scales"])
    y = M.moe_fused_ffn(r["x_perm"], r["expert_offsets"], W, x_perm_scales=r["x_perm_scales"])
    out2 = M.moe_combine(y, r["slot_of"], w)
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    assert torch.equal(out, out2)
    # the same scales on the power-of-two path are refused on the device
    Wp = M.Weights(wl.act, wl.wt, d["w1"], d["w2"], d["w1_scales"], d["w2_scales"])
    M.moe_forward(d["x"], d["logits"], Wp, wl.k, wl.score, bias=d["bias"], x_scales=d["x_scales"])
    st, site = M.moe_get_device_error()
    assert M.moe_status_string(st) == "MOE_ERR_UNSUPPORTED" and site == 301


def test_fp32_scales_on_power_of_two_inputs_match_fast_path():
    # power-of-two scales are a special case of fp32 scales: both paths agree to fp32 rounding
    wl = CASES["v3_fp8"]
    d = synth.make_inputs(wl, DEV)
    outs = []
    for fmt in ("pow2", "fp32"):
        W = M.Weights(wl.act, wl.wt, d["w1"], d["w2"], d["w1_scales"], d["w2_scales"],
                      scale_fmt=fmt)
        outs.append(M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, bias=d["bias"],
                                  x_scales=d["x_scales"]))
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    a, b = (host_values(o, None, "bf16") for o in outs)
    assert_parity(a, b, "bf16", 1e-2)
