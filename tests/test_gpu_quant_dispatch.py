"""The quantising dispatch (BF16 rows into an E4M3 layer) through the C ABI against the oracle:
codes and scales bit-exact, the permutation identical to the plain dispatch, and moe_forward
on BF16 input identical to moe_forward on the oracle's own quantisation of that input."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

M = pytest.importorskip("moe_expert_layer_prefix_b200")
DEV = "cuda"

SMALL = {
    "v3_fp8": synth.WORKLOADS["v3_fp8"].scaled(T=300, H=1024, E=16, k=4, I=512),
    "decode_fp8_fp4": synth.WORKLOADS["decode_fp8_fp4"].scaled(T=33, H=1024, E=64, I=256),
    "skewed_fp8_fp4": synth.WORKLOADS["skewed_fp8_fp4"].scaled(T=260, H=512, E=128, I=256),
}


@pytest.fixture(autouse=True)
def _clear_device_error():
    M.moe_get_device_error()
    yield


def _bf16_inputs(wl):
    d = synth.make_inputs(wl, DEV)
    xb = synth.make_activations(dataclasses.replace(wl, act="bf16"), DEV)["x"]
    return d, xb


def _bits(x_bf16):
    return x_bf16.view(torch.int16).cpu().numpy().view(np.uint16)


def _check_rows(r, codes, scales, k, slots):
    perm_src = r["perm_src"].cpu().numpy()
    xp = r["x_perm"].cpu().numpy()
    xps = r["x_perm_scales"].cpu().numpy()
    for p in slots:
        t = perm_src[p] // k
        assert np.array_equal(xp[p], codes[t]), p
        assert np.array_equal(xps[p], scales[t]), p


@pytest.mark.parametrize("name", list(SMALL))
def test_dispatch_quant_bit_exact(name):
    wl = SMALL[name]
    d, xb = _bf16_inputs(wl)
    idx, _ = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"])
    r = M.moe_dispatch_quant(xb, idx, wl.E)
    ref = M.moe_dispatch(xb, idx, wl.E, "bf16")
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    for key in ("expert_offsets", "perm_src", "slot_of"):
        assert torch.equal(r[key], ref[key]), key
    codes, scales = oracle.quantize_activations(_bits(xb))
    _check_rows(r, codes, scales, wl.k, range(wl.S))


def test_dispatch_quant_edges():
    """Zero blocks, exact 448 * 2^n boundaries, the largest and smallest BF16 magnitudes."""
    wl = SMALL["v3_fp8"].scaled(T=40)
    d, xb = _bf16_inputs(wl)
    x = xb.float()
    x[0, :128] = 0.0
    x[1, :] = 0.0
    x[2, 3] = 448.0 * 2 ** 5
    x[3, 130] = -448.0 * 2 ** 5 * (1 + 2 ** -7)
    x[4, :128] = 3.0e38
    x[5, :128] = 1.0e-38
    x[6, 256:384] = torch.linspace(-2e-30, 2e-30, 128)
    xb = x.to(torch.bfloat16)
    idx, _ = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"])
    r = M.moe_dispatch_quant(xb, idx, wl.E)
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    codes, scales = oracle.quantize_activations(_bits(xb))
    _check_rows(r, codes, scales, wl.k, range(wl.S))


def test_dispatch_quant_full_size_sampled():
    wl = synth.WORKLOADS["v3_fp8"]
    d, xb = _bf16_inputs(wl)
    idx, _ = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"])
    r = M.moe_dispatch_quant(xb, idx, wl.E)
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    rng = np.random.default_rng(5)
    tokens = rng.choice(wl.T, size=64, replace=False)
    codes, scales = oracle.quantize_activations(_bits(xb[torch.as_tensor(tokens, device=DEV)]))
    slot_of = r["slot_of"].cpu().numpy().reshape(wl.T, wl.k)
    xp = r["x_perm"].cpu().numpy()
    xps = r["x_perm_scales"].cpu().numpy()
    for i, t in enumerate(tokens):
        for j in range(wl.k):
            p = slot_of[t, j]
            assert np.array_equal(xp[p], codes[i]) and np.array_equal(xps[p], scales[i])


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_bf16_input_equals_prequantised(name):
    wl = SMALL[name]
    d, xb = _bf16_inputs(wl)
    W = M.Weights(wl.act, wl.wt, d["w1"], d["w2"], d["w1_scales"], d["w2_scales"])
    a = M.moe_forward(xb, d["logits"], W, wl.k, wl.score, bias=d["bias"], renorm=wl.renorm)
    codes, scales = oracle.quantize_activations(_bits(xb))
    xq = torch.from_numpy(codes).to(DEV)
    xs = torch.from_numpy(scales).to(DEV)
    b = M.moe_forward(xq, d["logits"], W, wl.k, wl.score, bias=d["bias"], renorm=wl.renorm,
                      x_scales=xs)
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    assert torch.equal(a, b)
