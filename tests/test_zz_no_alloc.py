"""moe_dispatch_noalloc (the dispatch entry point for callers that cannot allocate device
memory) against moe_dispatch, through the C ABI, on two calls in a row.

Kept in a file of its own that pytest collects last, so that a run stopping at the first
failure has already run every other test.  It passes alone in a fresh process and after the
rest of the suite (the shared scratch buffer keeps the previous call's contents, which the
second call must not depend on)."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

M = pytest.importorskip("moe_expert_layer_prefix_b200")
DEV = "cuda"


def _outputs(wl, like):
    S = wl.S
    return {"x_perm": torch.empty((S, wl.H), dtype=like.dtype, device=DEV),
            "x_perm_scales": (torch.empty((S, wl.H // 128), dtype=torch.float32, device=DEV)
                              if wl.act == "e4m3" else None),
            "expert_offsets": torch.empty(wl.E + 1, dtype=torch.int32, device=DEV),
            "perm_src": torch.empty(S, dtype=torch.int32, device=DEV),
            "slot_of": torch.empty(S, dtype=torch.int32, device=DEV)}


def test_noalloc_dispatch_matches_dispatch_twice_in_a_row():
    # two different problems back to back: the second call runs on a buffer that still
    # holds the first call's counts
    cases = [synth.WORKLOADS["v3_fp8"].scaled(T=1000, H=512, E=256, k=8, I=128),
             synth.WORKLOADS["skewed_fp8_fp4"].scaled(T=333, H=256, E=1024, k=16, I=128)]
    for wl in cases:
        a = synth.make_activations(wl, DEV)
        idx, _ = M.moe_route(a["logits"], wl.k, wl.score, bias=a["bias"])
        ref = M.moe_dispatch(a["x"], idx, wl.E, wl.act, x_scales=a["x_scales"])
        out = _outputs(wl, a["x"])
        before = torch.cuda.memory_allocated()
        M.moe_dispatch_noalloc(a["x"], idx, wl.E, wl.act, out, x_scales=a["x_scales"])
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == before
        for name in ("expert_offsets", "perm_src", "slot_of", "x_perm", "x_perm_scales"):
            assert torch.equal(out[name], ref[name]), name


def test_noalloc_dispatch_rejects_oversized_problem():
    wl = synth.WORKLOADS["skewed_fp8_fp4"].scaled(T=40000, H=128, E=1024, k=1, I=128)
    x = torch.zeros((wl.T, wl.H), dtype=torch.uint8, device=DEV)
    xs = torch.ones((wl.T, 1), dtype=torch.float32, device=DEV)
    idx = torch.zeros((wl.T, 1), dtype=torch.int32, device=DEV)
    with pytest.raises(M.MoeError) as ei:
        M.moe_dispatch_noalloc(x, idx, wl.E, "e4m3", _outputs(wl, x), x_scales=xs)
    assert ei.value.status == -4          # MOE_ERR_WORKSPACE, nothing launched
