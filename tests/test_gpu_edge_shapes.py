"""The whole layer at the degenerate shapes the method has, against the oracle and against the
unfused chain: the smallest hidden and intermediate sizes the ABI accepts (H = I = 128, one
K-step per tile), a single expert (the dense FFN), every expert picked by every token
(k = E) and a single token."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.util import TOL, assert_parity, host_values, oracle_layer, weights_of

pytestmark = pytest.mark.gpu

M = pytest.importorskip("moe_expert_layer_prefix_b200")
DEV = "cuda"

W_ = synth.WORKLOADS
EDGE = {
    "v3_fp8_h128_i128": W_["v3_fp8"].scaled(T=50, H=128, E=4, k=2, I=128),
    "decode_fp8_fp4_h128_i128_k_eq_E": W_["decode_fp8_fp4"].scaled(T=9, H=128, E=8, k=8,
                                                                   I=128),
    "mixtral_bf16_h128_i128": W_["mixtral_bf16"].scaled(T=40, H=128, E=3, k=2, I=128),
    "v3_fp8_one_expert": W_["v3_fp8"].scaled(T=70, H=256, E=1, k=1, I=256),
    "mixtral_bf16_one_expert": W_["mixtral_bf16"].scaled(T=70, H=256, E=1, k=1, I=256),
    "decode_fp8_fp4_T1": W_["decode_fp8_fp4"].scaled(T=1, H=512, E=16, k=8, I=256),
    "skewed_fp8_fp4_T1": W_["skewed_fp8_fp4"].scaled(T=1, H=256, E=64, k=16, I=128),
    # E2M1 weights: the GEMM's stager warp runs for K loops of 8 or more 128-deep k-steps
    # only, so in the persistent kernel one GEMM phase takes it and the other does not
    "decode_fp8_fp4_short_then_long_k": W_["decode_fp8_fp4"].scaled(T=24, H=512, E=8, k=4,
                                                                    I=1024),
    "skewed_fp8_fp4_long_then_short_k": W_["skewed_fp8_fp4"].scaled(T=40, H=1024, E=16, k=4,
                                                                    I=512),
}


@pytest.fixture(autouse=True)
def _clean():
    M.moe_get_device_error()
    yield
    M.moe_set_gemm_tiles("auto")


@pytest.mark.parametrize("name,tiles",
                         [(n, t) for n in EDGE for t in ("auto", "single", "small", "pair")])
def test_forward_matches_oracle(name, tiles):
    wl = EDGE[name]
    d = synth.make_inputs(wl, DEV)
    W = weights_of(wl, d)
    M.moe_set_gemm_tiles(tiles)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device=DEV)
    out = M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, bias=d["bias"],
                        renorm=wl.renorm, x_scales=d["x_scales"], topk_idx=idx)
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    r = oracle.forward(oracle_layer(wl, d), return_all=True)
    assert np.array_equal(idx.cpu().numpy(), r["topk_idx"])
    fmt = "f32" if wl.act == "f32" else "bf16"
    assert_parity(host_values(out, None, fmt), r["out"], fmt, TOL[wl.act])


@pytest.mark.parametrize("tiles", ["single", "small", "pair"])
@pytest.mark.parametrize("name", list(EDGE))
def test_forward_equals_unfused_chain(name, tiles):
    wl = EDGE[name]
    d = synth.make_inputs(wl, DEV)
    W = weights_of(wl, d)
    M.moe_set_gemm_tiles(tiles)
    out = M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, bias=d["bias"],
                        renorm=wl.renorm, x_scales=d["x_scales"])
    idx, w = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"], renorm=wl.renorm)
    r = M.moe_dispatch(d["x"], idx, wl.E, wl.act, x_scales=d["x_scales"])
    y = M.moe_fused_ffn(r["x_perm"], r["expert_offsets"], W, x_perm_scales=r["x_perm_scales"])
    out2 = M.moe_combine(y, r["slot_of"], w)
    torch.cuda.synchronize()
    assert M.moe_get_device_error()[0] == 0
    assert torch.equal(out, out2)
