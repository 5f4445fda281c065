"""Group-limited routing with a routed scaling factor through the C ABI against the oracle:
indices bit-exact, gates within 1e-6 relative; moe_forward_ex equal to the chain routed the
same way; invalid configurations rejected before any launch."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

M = pytest.importorskip("moe_expert_layer_prefix_b200")
DEV = "cuda"


@pytest.fixture(autouse=True)
def _clear_device_error():
    M.moe_get_device_error()
    yield


CASES = [  # (score, T, E, k, n_group, topk_group, scale, bias)
    ("sigmoid", 2048, 256, 8, 8, 4, 2.5, True),     # V3-style
    ("softmax", 1000, 1024, 16, 8, 3, 1.0, False),
    ("softmax", 777, 64, 6, 2, 1, 0.5, False),
    ("sigmoid", 300, 512, 32, 4, 4, 1.0, True),     # all groups kept: plain routing
    ("sigmoid", 64, 1024, 1, 32, 1, 3.0, False),    # one expert from the single best group
]


@pytest.mark.parametrize("case", CASES)
def test_route_groups_bit_exact(case):
    score, T, E, k, ng, tg, scale, with_bias = case
    g = torch.Generator(device=DEV).manual_seed(T + E)
    logits = torch.randn((T, E), generator=g, device=DEV)
    logits[::4] = torch.round(logits[::4] * 2) / 2          # equal keys and group scores
    bias = (torch.randn(E, generator=g, device=DEV) * 0.1) if with_bias else None
    idx, w = M.moe_route(logits, k, score, bias=bias, groups=(ng, tg, scale))
    torch.cuda.synchronize()
    ridx, rw = oracle.route(logits.cpu().numpy(), None if bias is None else bias.cpu().numpy(),
                            k, score, True, n_group=ng, topk_group=tg, scale=scale)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.max(np.abs(w.cpu().numpy() - rw) / np.abs(rw)) < 1e-6


@pytest.mark.parametrize("name", ["v3_fp8", "skewed_fp8_fp4"])
def test_forward_groups_equals_chain(name):
    wl = synth.WORKLOADS[name].scaled(T=256, H=512, I=256)
    groups = (8, 3, 2.0)
    d = synth.make_inputs(wl, DEV)
    W = M.Weights(wl.act, wl.wt, d["w1"], d["w2"], d["w1_scales"], d["w2_scales"])
    idx1 = torch.empty((wl.T, wl.k), dtype=torch.int32, device=DEV)
    out = M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, bias=d["bias"],
                        renorm=wl.renorm, x_scales=d["x_scales"], topk_idx=idx1, groups=groups)
    idx, w = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"], renorm=wl.renorm,
                         groups=groups)
    r = M.moe_dispatch(d["x"], idx, wl.E, wl.act, x_scales=d["x_scales"])
    y = M.moe_fused_ffn(r["x_perm"], r["expert_offsets"], W, x_perm_scales=r["x_perm_scales"])
    out2 = M.moe_combine(y, r["slot_of"], w)
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    assert torch.equal(idx1, idx)
    assert torch.equal(out, out2)
    ridx, _ = oracle.route(d["logits"].cpu().numpy(),
                           None if d["bias"] is None else d["bias"].cpu().numpy(), wl.k,
                           wl.score, wl.renorm, n_group=8, topk_group=3, scale=2.0)
    assert np.array_equal(idx.cpu().numpy(), ridx)


@pytest.mark.parametrize("groups,status", [((3, 1, 1.0), "MOE_ERR_UNSUPPORTED"),   # 256 % 3
                                           ((16, 2, 1.0), "MOE_ERR_UNSUPPORTED"),  # G = 16
                                           ((8, 9, 1.0), "MOE_ERR_INVALID_ARG"),   # > n_group
                                           ((8, 0, 1.0), "MOE_ERR_INVALID_ARG"),
                                           ((0, 1, 1.0), "MOE_ERR_INVALID_ARG"),
                                           ((8, 1, float("nan")), "MOE_ERR_INVALID_ARG")])
def test_route_groups_invalid(groups, status):
    logits = torch.zeros((4, 256), device=DEV)
    with pytest.raises(M.MoeError) as ei:
        M.moe_route(logits, 8, "softmax", groups=groups)
    assert status in str(ei.value)


def test_route_groups_too_few_experts_kept():
    logits = torch.zeros((4, 256), device=DEV)
    with pytest.raises(M.MoeError) as ei:
        M.moe_route(logits, 33, "softmax", groups=(8, 1, 1.0))   # k > 1 * 32 (and k > 32)
    assert "MOE_ERR" in str(ei.value)
