"""moe_dispatch_noalloc (the dispatch entry point for callers that cannot allocate device
memory) against moe_dispatch, through the C ABI, on two calls in a row.

Kept in a file of its own that pytest collects last, so that a run stopping at the first
failure has already run every other test.  It passes alone in a fresh process and after the
rest of the suite (the shared scratch buffer keeps the previous call's contents, which the
second call must not depend on).

Callers of this entry point cannot allocate device memory (a plain C host with no device
allocator of its own, a runtime that plans every device byte at start-up, or a path where
cudaMalloc / cudaFree would synchronise the device), so the tests also check that the call
itself allocates nothing and that the size limit of the built-in 4 MiB scratch is exact."""
import ctypes

import pytest
import torch

import synth

M = pytest.importorskip("moe_expert_layer_prefix_b200")
DEV = "cuda"
gpu = pytest.mark.gpu

# the largest T whose dispatch workspace fits the 4 MiB scratch at E = 1024:
# ceil(T / 32) * 1024 * 4 bytes of chunk counts + 1024 * 4 bytes of totals <= 4 MiB
T_MAX_E1024 = 32736


def _outputs(wl, like):
    S = wl.S
    return {"x_perm": torch.empty((S, wl.H), dtype=like.dtype, device=DEV),
            "x_perm_scales": (torch.empty((S, wl.H // 128), dtype=torch.float32, device=DEV)
                              if wl.act == "e4m3" else None),
            "expert_offsets": torch.empty(wl.E + 1, dtype=torch.int32, device=DEV),
            "perm_src": torch.empty(S, dtype=torch.int32, device=DEV),
            "slot_of": torch.empty(S, dtype=torch.int32, device=DEV)}


@gpu
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


@gpu
def test_noalloc_dispatch_rejects_oversized_problem():
    wl = synth.WORKLOADS["skewed_fp8_fp4"].scaled(T=40000, H=128, E=1024, k=1, I=128)
    x = torch.zeros((wl.T, wl.H), dtype=torch.uint8, device=DEV)
    xs = torch.ones((wl.T, 1), dtype=torch.float32, device=DEV)
    idx = torch.zeros((wl.T, 1), dtype=torch.int32, device=DEV)
    with pytest.raises(M.MoeError) as ei:
        M.moe_dispatch_noalloc(x, idx, wl.E, "e4m3", _outputs(wl, x), x_scales=xs)
    assert ei.value.status == -4          # MOE_ERR_WORKSPACE, nothing launched


def test_noalloc_size_limit_is_exact_on_the_host():
    # refused before anything touches a device: T_MAX + 1 tokens at E = 1024 need 4 KiB
    # more than the scratch holds; the dummy addresses are never dereferenced
    fake = ctypes.c_void_p(1 << 20)
    assert M.moe_workspace_size("dispatch", T_MAX_E1024, 128, 1024, 1, 128, "e4m3",
                                "e4m3") == 4 << 20
    st = M._dispatch_noalloc(fake, fake, 2, T_MAX_E1024 + 1, 128, 1024, 1, fake, fake, fake,
                             fake, fake, fake, None)
    assert M.moe_status_string(st) == "MOE_ERR_WORKSPACE"
    # shapes moe_dispatch does not support give moe_dispatch's status, not a size error
    st = M._dispatch_noalloc(fake, fake, 2, 4, 128, 1025, 1, fake, fake, fake, fake, fake,
                             fake, None)
    assert M.moe_status_string(st) == "MOE_ERR_UNSUPPORTED"
    st = M._dispatch_noalloc(fake, fake, 2, 4, 128, 64, 33, fake, fake, fake, fake, fake,
                             fake, None)
    assert M.moe_status_string(st) == "MOE_ERR_UNSUPPORTED"
    st = M._dispatch_noalloc(fake, fake, 2, 0, 128, 64, 2, fake, fake, fake, fake, fake,
                             fake, None)
    assert M.moe_status_string(st) == "MOE_ERR_INVALID_ARG"


@gpu
def test_noalloc_dispatch_at_the_size_limit_and_bf16():
    # the largest accepted problem at E = 1024 (scratch filled to the last byte), then a
    # BF16 problem, each against moe_dispatch
    cases = [synth.WORKLOADS["skewed_fp8_fp4"].scaled(T=T_MAX_E1024, H=128, E=1024, k=2,
                                                      I=128),
             synth.WORKLOADS["mixtral_bf16"].scaled(T=777, H=384, E=8, k=2, I=128)]
    for wl in cases:
        a = synth.make_activations(wl, DEV)
        idx, _ = M.moe_route(a["logits"], wl.k, wl.score, bias=a["bias"])
        ref = M.moe_dispatch(a["x"], idx, wl.E, wl.act, x_scales=a["x_scales"])
        out = _outputs(wl, a["x"])
        before = torch.cuda.memory_allocated()
        M.moe_dispatch_noalloc(a["x"], idx, wl.E, wl.act, out, x_scales=a["x_scales"])
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == before
        assert M.moe_get_device_error()[0] == 0
        for name in ("expert_offsets", "perm_src", "slot_of", "x_perm", "x_perm_scales"):
            assert (out[name] is None and ref[name] is None) or torch.equal(out[name],
                                                                           ref[name]), name
