"""Backward of the BF16 layer through the C ABI (moe_transpose_experts, moe_expert_backward)
against the oracle's backward evaluated with the same storage points
(oracle.backward.layer_backward_stored).

Tolerance: the GPU takes each BF16 storage decision on its fp32 value, the oracle on its fp64
value, so single elements of dh, dG, dx_slot (and of the forward's h, y) may land one BF16
step apart and carry that into later sums.  An fp32 emulation of the GPU's arithmetic
against the stored oracle gives max(|d| - ulp) / rms <= 7.7e-3 and rel-L2 <= 2.4e-4 for every
gradient on these shapes; the test allows rel-L2 2e-3 everywhere and max 2e-2 for dx and
d logits.  A weight-gradient entry sums only its expert's n_e rows, so one BF16 step in one
large stored dG (or dy_w, h) element moves it by 2^-8 |dG| |x| against an rms of about
sqrt(n_e) rms(dG) rms(x), up to 2^-8 * 27 / 2 = 5.3e-2 with |dG| <= 6 rms, |x| <= 4.5 rms
and n_e ~ 4 (the small-tile case).  That step is allowed explicitly, from the oracle's own
stored values, to first order: dG itself may move by one step of its own and by the step of
the stored dh it was computed from (dg and du are linear in dh, so by |dG| ulp(dh) / |dh|);
for dW1_e the sum over the expert's rows of that times |x|, for dW2_e of
ulp(dy_w) x |h| + |dy_w| x ulp(h) (the weight gradients themselves are fp32 sums of exact
products).  What remains must stay under 2e-2, as for dx."""
import numpy as np
import pytest
import torch

import synth
from oracle import backward as B
from tests.util import host_values, oracle_layer, parity_err, store_ulp, weights_of

pytestmark = pytest.mark.gpu

M = pytest.importorskip("moe_expert_layer_prefix_b200")
DEV = "cuda"
MAX_TOL = {"dx": 2e-2, "dlogits": 2e-2, "dw1": 2e-2, "dw2": 2e-2}
L2_TOL = 2e-3

W_ = synth.WORKLOADS["mixtral_bf16"]
CASES = {
    "softmax": W_.scaled(T=200, H=512, E=8, I=256),
    "softmax_no_renorm": W_.scaled(T=100, H=256, E=5, k=2, I=128, renorm=False),
    "sigmoid_bias": W_.scaled(T=150, H=384, E=6, k=3, I=256, score="sigmoid", bias=True),
    "pair_tiles": W_.scaled(T=600, H=256, E=4, k=2, I=128),          # >= 128 rows per expert
    "small_tiles": W_.scaled(T=64, H=256, E=64, k=4, I=128),         # <= 16 rows per expert
}


@pytest.mark.parametrize("dtype,shape", [(torch.bfloat16, (3, 70, 129)),
                                         (torch.float32, (2, 64, 32)),
                                         (torch.uint8, (5, 33, 31)),
                                         (torch.bfloat16, (8, 512, 256))])
def test_transpose_bit_exact(dtype, shape):
    g = torch.Generator(device=DEV).manual_seed(1)
    if dtype == torch.uint8:
        src = torch.randint(0, 256, shape, dtype=torch.uint8, device=DEV, generator=g)
    else:
        src = torch.randn(shape, generator=g, device=DEV).to(dtype)
    out = M.moe_transpose_experts(src)
    torch.cuda.synchronize()
    assert torch.equal(out, src.transpose(1, 2).contiguous())


def _backward(wl, d, dout):
    W = weights_of(wl, d)
    idx, w = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"], renorm=wl.renorm)
    r = M.moe_dispatch(d["x"], idx, wl.E, wl.act)
    h, _ = M.moe_expert_linear1(r["x_perm"], r["expert_offsets"], W)
    y = M.moe_expert_linear2(h, r["expert_offsets"], W)
    w1_t = M.moe_transpose_experts(W.w1)
    w2_t = M.moe_transpose_experts(W.w2)
    g = M.moe_expert_backward(dout, d["logits"], idx, w, r["expert_offsets"], r["slot_of"],
                              r["x_perm"], h, y, W, w1_t, w2_t, wl.k, wl.score, wl.renorm)
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    return idx, g


def _weight_grad_allowance(ref):
    """One BF16 step at each stored per-slot value a weight gradient sums (module docstring),
    per expert, in the weight gradients' shapes."""
    sl, offs = ref["slots"], ref["offsets"]
    u = {n: store_ulp(sl[n], "bf16") for n in ("dG", "dy_w", "h", "dh")}
    dh = np.abs(sl["dh"])
    rel_dh = np.where(dh > 0, u["dh"] / np.where(dh > 0, dh, 1.0), 0.0)
    # dG's movement: its own step plus the step of dh (both halves depend on the same dh)
    mv_dG = u["dG"] + np.abs(sl["dG"]) * np.concatenate([rel_dh, rel_dh], axis=1)
    a1 = np.zeros_like(ref["dw1"])
    a2 = np.zeros_like(ref["dw2"])
    for e in range(len(offs) - 1):
        a, b = int(offs[e]), int(offs[e + 1])
        if a == b:
            continue
        a1[e] = mv_dG[a:b].T @ np.abs(sl["x"][a:b])
        a2[e] = u["dy_w"][a:b].T @ np.abs(sl["h"][a:b]) + np.abs(sl["dy_w"][a:b]).T @ u["h"][a:b]
    return {"dw1": a1, "dw2": a2}


def _dout(wl):
    g = torch.Generator(device=DEV).manual_seed(7)
    return torch.randn((wl.T, wl.H), generator=g, device=DEV).to(torch.bfloat16)


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(name):
    wl = CASES[name]
    d = synth.make_inputs(wl, DEV)
    dout = _dout(wl)
    idx, got = _backward(wl, d, dout)
    ref = B.layer_backward_stored(oracle_layer(wl, d), host_values(dout, None, "bf16"),
                                  return_slots=True)
    assert np.array_equal(idx.cpu().numpy(), ref["topk_idx"])
    allow = _weight_grad_allowance(ref)
    for n in ("dx", "dw1", "dw2", "dlogits"):
        fmt = "bf16" if n == "dx" else "f32"
        v = host_values(got[n], None, fmt)
        mx, l2 = parity_err(v, ref[n], fmt, allow=allow.get(n))
        assert mx <= MAX_TOL[n] and l2 <= L2_TOL, (n, mx, l2)
    # experts no token picked get exactly zero weight gradients
    picked = np.zeros(wl.E, bool)
    picked[np.unique(ref["topk_idx"])] = True
    assert not torch.any(got["dw1"][torch.from_numpy(~picked).to(DEV)])


def test_backward_deterministic():
    wl = CASES["sigmoid_bias"]
    d = synth.make_inputs(wl, DEV)
    dout = _dout(wl)
    _, a = _backward(wl, d, dout)
    _, b = _backward(wl, d, dout)
    for n in a:
        assert torch.equal(a[n], b[n]), n
