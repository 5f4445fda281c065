"""Failure detection on the GPU without a fault: every wait in the library's kernels is
bounded.  A self-test kernel waits on a barrier that can never complete, by construction
(an mbarrier nothing arrives on; a grid barrier expecting one arrival more than the grid
has).  With a short wait limit the wait must give up, record MOE_ERR_TIMEOUT with its site
in the device error word, and return, after which the same context runs the layer
correctly.  Nothing traps, faults or waits without a limit."""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.util import TOL, assert_parity, host_values, oracle_layer, weights_of

pytestmark = pytest.mark.gpu

M = pytest.importorskip("moe_expert_layer_prefix_b200")
DEV = "cuda"
LIMIT = 2_000_000          # SM clock cycles: about 1 ms at 2 GHz


def _layer_ok():
    wl = synth.WORKLOADS["v3_fp8"].scaled(T=96, H=512, E=16, k=4, I=256)
    d = synth.make_inputs(wl, DEV)
    out = M.moe_forward(d["x"], d["logits"], weights_of(wl, d), wl.k, wl.score,
                        bias=d["bias"], x_scales=d["x_scales"])
    st, site = M.moe_get_device_error()
    assert st == 0, (st, site)
    assert_parity(host_values(out, None, "bf16"), oracle.forward(oracle_layer(wl, d)), "bf16",
                  TOL[wl.act])


@pytest.mark.parametrize("kind,site", [("mbarrier", 901), ("grid_barrier", 201)])
def test_bounded_wait_runs_out_and_reports(kind, site):
    M.moe_get_device_error()                      # start from a clear error word
    _layer_ok()                                   # and a working context
    M.moe_set_wait_limit(LIMIT)
    try:
        torch.cuda.synchronize()
        t = time.perf_counter()
        M.moe_selftest_wait(kind)
        st, got_site = M.moe_get_device_error()   # synchronises: the kernel has returned
        dt = time.perf_counter() - t
    finally:
        M.moe_set_wait_limit(0)
    assert M.moe_status_string(st) == "MOE_ERR_TIMEOUT"
    assert got_site == site
    # it gave up after the short limit, not the default one of about a second
    assert dt < 0.5, dt
    # the error word was cleared by the read, and the context still computes the layer
    assert M.moe_get_device_error()[0] == 0
    _layer_ok()


def test_default_wait_limit_restored_for_normal_work():
    # a limit of zero restores the default; a full layer of many tiles then runs clean
    M.moe_set_wait_limit(0)
    wl = synth.WORKLOADS["skewed_fp8_fp4"].scaled(T=512, H=512, E=32, k=8, I=256)
    d = synth.make_inputs(wl, DEV)
    M.moe_forward(d["x"], d["logits"], weights_of(wl, d), wl.k, wl.score,
                  x_scales=d["x_scales"])
    assert M.moe_get_device_error()[0] == 0
