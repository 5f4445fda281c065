"""fp32 block scales must be positive normal powers of two (the tensor cores consume them as
UE8M0 exponent bytes).  A GEMM that reads any other scale records MOE_ERR_UNSUPPORTED at the
scale-format site in the device error word; power-of-two scales record nothing."""
import pytest
import torch

import synth
from tests.util import weights_of

pytestmark = pytest.mark.gpu

M = pytest.importorskip("moe_expert_layer_prefix_b200")
DEV = "cuda"
SITE_SCALE_FORMAT = 301
UNSUPPORTED = -2

CASES = {
    "v3_fp8": synth.WORKLOADS["v3_fp8"].scaled(T=300, H=1024, E=16, k=4, I=512),
    "decode_fp8_fp4": synth.WORKLOADS["decode_fp8_fp4"].scaled(T=33, H=1024, E=64, I=256),
}


def _run(wl, d, api):
    W = weights_of(wl, d)
    M.moe_get_device_error()
    if api == "forward":
        M.moe_forward(d["x"], d["logits"], W, wl.k, wl.score, bias=d["bias"],
                      renorm=wl.renorm, x_scales=d["x_scales"])
    else:
        idx, _ = M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"])
        r = M.moe_dispatch(d["x"], idx, wl.E, wl.act, x_scales=d["x_scales"])
        M.moe_fused_ffn(r["x_perm"], r["expert_offsets"], W, x_perm_scales=r["x_perm_scales"])
    torch.cuda.synchronize()
    return M.moe_get_device_error()


@pytest.mark.parametrize("api", ["forward", "chain"])
@pytest.mark.parametrize("name", list(CASES))
def test_pow2_scales_record_nothing(name, api):
    wl = CASES[name]
    assert _run(wl, synth.make_inputs(wl, DEV), api) == (0, 0)


@pytest.mark.parametrize("api", ["forward", "chain"])
@pytest.mark.parametrize("value", [1.5, -1.0, 0.0, float("inf"), 2.0 ** -127])
@pytest.mark.parametrize("name", list(CASES))
def test_bad_activation_scale_recorded(name, value, api):
    wl = CASES[name]
    d = synth.make_inputs(wl, DEV)
    d["x_scales"][wl.T // 2, 1] = value      # every slot of that token reads it
    assert _run(wl, d, api) == (UNSUPPORTED, SITE_SCALE_FORMAT)


@pytest.mark.parametrize("api", ["forward", "chain"])
@pytest.mark.parametrize("which", ["w1_scales", "w2_scales"])
def test_bad_weight_scale_recorded(which, api):
    wl = CASES["v3_fp8"]
    d = synth.make_inputs(wl, DEV)
    d[which][:, 0, 0] *= 1.5                 # block (0, 0) of every expert
    assert _run(wl, d, api) == (UNSUPPORTED, SITE_SCALE_FORMAT)
    # the error word was cleared by the read: the next clean call records nothing
    assert _run(wl, synth.make_inputs(wl, DEV), api) == (0, 0)
