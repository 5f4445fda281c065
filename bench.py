"""Benchmark of the fused MoE expert layer on B200 -- one JSON line on stdout (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

A step is one pass of the whole layer (route -> dispatch -> linear-1 + SwiGLU + requant ->
linear-2 -> combine) over one batch of seeded synthetic input, through the library's C ABI.
The default workload is the DeepSeek-V3-shaped FP8 layer (T=8192, H=7168, E=256, top-8,
I=2048).  Inputs are resident in HBM when the timed region starts; the 11 GB of expert
weights read per step are far larger than the 126 MB L2, so no flush is needed.

Multi-GPU: the layer does not shard here (no collective on the data path), so N ranks run
N independent replicas ("scaling": "weak"); time is the max over ranks.

--impl reference times the CPU oracle on this host (rank 0 only) on a bounded token
sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}

# DRAM traffic of a kernel as a multiple of its algorithmic bytes, from an ncu capture of a
# smaller case with the same rows per expert (dram__bytes_read.sum + dram__bytes_write.sum
# of one launch).  Used for the roofline's "traffic".
TRAFFIC_RATIO = {
    ("v3_fp8", "linear1"): (1.022, "the V3-shaped layer at T=1024, E=32"),
    ("v3_fp8", "linear2"): (0.964, "the V3-shaped layer at T=1024, E=32"),
    ("decode_fp8_fp4", "linear1"): (1.013, "the decode-shaped layer at E=64"),
}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1 and args.impl == "reference":
        return ws, rank, local          # rank 0 alone runs the oracle; no process group
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if (args.impl == "native" and torch.cuda.is_available()) else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def max_over_ranks(v: float, ws: int) -> float:
    if ws == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons while the GPU is busy."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def workload(args) -> synth.Workload:
    """The named workload, optionally shrunk (--T/--E) for a profiling capture."""
    wl = synth.WORKLOADS[args.workload]
    over = {n: v for n, v in (("T", args.T), ("E", args.E)) if v is not None}
    if over:
        wl = wl.scaled(name=wl.name + "_" + "_".join(f"{n}{v}" for n, v in over.items()), **over)
    return wl


def algorithmic(wl: synth.Workload, touched: int):
    """Algorithmic bytes / FLOPs per stage (one launch of each stage per step)."""
    T, H, E, k, I, S = wl.T, wl.H, wl.E, wl.k, wl.I, wl.S
    a = {"f32": 4, "bf16": 2, "e4m3": 1}[wl.act]
    if wl.wt == "e2m1":
        w1 = 2 * I * H * (0.5 + 1 / 32)
        w2 = H * I * (0.5 + 1 / 32)
    elif wl.wt == "e4m3":
        w1 = 2 * I * H + (2 * I // 128) * (H // 128) * 4
        w2 = H * I + (H // 128) * (I // 128) * 4
    else:
        wb = {"bf16": 2, "f32": 4}[wl.wt]
        w1, w2 = 2 * I * H * wb, H * I * wb
    xs = (H // 128) * 4 if wl.act == "e4m3" else 0
    hs = (I // 128) * 4 if wl.act == "e4m3" else 0
    ob = 4 if wl.act == "f32" else 2
    return {
        "route": {"bytes": T * E * 4 + T * k * 8, "flops": 0},
        "dispatch": {"bytes": T * (H * a + xs) + S * (H * a + xs) + S * 12, "flops": 0},
        "linear1": {"bytes": touched * w1 + S * (H * a + xs) + S * (I * a + hs),
                    "flops": 2.0 * S * H * 2 * I},
        "linear2": {"bytes": touched * w2 + S * (I * a + hs) + S * H * ob,
                    "flops": 2.0 * S * I * H},
        "combine": {"bytes": S * H * ob + T * H * ob + T * k * 8, "flops": 0},
    }


def run_native(args, ws, rank, local):
    import moe_expert_layer_prefix_b200 as M

    wl = workload(args)
    M.moe_set_gemm_tiles(args.tiles)
    dev = torch.device("cuda", torch.cuda.current_device())
    d = synth.make_inputs(wl, dev)
    if args.bf16_input:
        # BF16 activations into the E4M3 layer: the dispatch quantises them
        if wl.act != "e4m3":
            raise SystemExit("--bf16-input needs a workload with E4M3 activations")
        d["x"] = synth.make_activations(dataclasses.replace(wl, act="bf16"), dev)["x"]
        d["x_scales"] = None
    if args.scale_fmt == "fp32":
        # arbitrary fp32 block scales: the power-of-two scales times seeded factors in
        # [1.05, 1.95] (no scale stays a power of two)
        if wl.act != "e4m3" or wl.wt != "e4m3":
            raise SystemExit("--scale-fmt fp32 needs E4M3 activations and weights")
        g = torch.Generator(device=dev).manual_seed(1234)
        for n in ("x_scales", "w1_scales", "w2_scales"):
            d[n] = (d[n] * (1.05 + 0.9 * torch.rand(d[n].shape, generator=g, device=dev))).contiguous()
    W = M.Weights(wl.act, wl.wt, d["w1"], d["w2"], d["w1_scales"], d["w2_scales"],
                  scale_fmt=args.scale_fmt)
    T, H, E, k, I, S = wl.T, wl.H, wl.E, wl.k, wl.I, wl.S
    stream = torch.cuda.current_stream()

    # buffers of the unfused chain (each call is one C-ABI entry point)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gw = torch.empty((T, k), dtype=torch.float32, device=dev)
    xdt = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}[wl.act]
    disp = {"x_perm": torch.empty((S, H), dtype=xdt, device=dev),
            "x_perm_scales": (torch.empty((S, H // 128), dtype=torch.float32, device=dev)
                              if wl.act == "e4m3" else None),
            "expert_offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
            "perm_src": torch.empty(S, dtype=torch.int32, device=dev),
            "slot_of": torch.empty(S, dtype=torch.int32, device=dev)}
    dws = M.workspace(M.moe_workspace_size("dispatch", T, H, E, k, I, wl.act, wl.wt), dev)
    hdt = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}[wl.act]
    h = torch.empty((S, I), dtype=hdt, device=dev)
    hs = torch.empty((S, I // 128), dtype=torch.float32, device=dev) if wl.act == "e4m3" else None
    ydt = torch.float32 if wl.act == "f32" else torch.bfloat16
    y = torch.empty((S, H), dtype=ydt, device=dev)
    out = torch.empty((T, H), dtype=ydt, device=dev)

    names = ["route", "dispatch", "linear1", "linear2", "combine"]

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        M.moe_route(d["logits"], k, wl.score, bias=d["bias"], renorm=wl.renorm, topk_idx=idx,
                    topk_w=gw, stream=stream)
        mark(1)
        if args.bf16_input:
            M.moe_dispatch_quant(d["x"], idx, E, ws=dws, out=disp, stream=stream)
        else:
            M.moe_dispatch(d["x"], idx, E, wl.act, x_scales=d["x_scales"], ws=dws, out=disp,
                           stream=stream)
        mark(2)
        M.moe_expert_linear1(disp["x_perm"], disp["expert_offsets"], W,
                             x_perm_scales=disp["x_perm_scales"], h=h, h_scales=hs,
                             stream=stream)
        mark(3)
        M.moe_expert_linear2(h, disp["expert_offsets"], W, h_scales=hs, y=y, stream=stream)
        mark(4)
        M.moe_combine(y, disp["slot_of"], gw, out=out, stream=stream)
        mark(5)

    fws = M.workspace(M.moe_workspace_size("forward", T, H, E, k, I, wl.act, wl.wt), dev)

    def fused_step():
        M.moe_forward(d["x"], d["logits"], W, k, wl.score, bias=d["bias"], renorm=wl.renorm,
                      x_scales=d["x_scales"], out=out, ws=fws, stream=stream)

    for _ in range(args.warmup):
        step()
        fused_step()
    torch.cuda.synchronize()
    st, site = M.moe_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error {M.moe_status_string(st)} at site {site}")
    counts = np.diff(disp["expert_offsets"].cpu().numpy())
    touched = int((counts > 0).sum())

    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    # (1) the headline step: moe_forward, one persistent launch per step
    barrier(ws)
    torch.cuda.synchronize()
    n0 = M.moe_launch_count()
    t0.record(stream)
    for i in range(args.steps):
        fused_step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    launches = M.moe_launch_count() - n0
    ms_total = max_over_ranks(t0.elapsed_time(t1), ws)
    ms = ms_total / args.steps
    # (2) the same layer as the chain of entry points, CUDA events between the calls
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    chain_ms = max_over_ranks(t0.elapsed_time(t1), ws) / args.steps
    clk = clocks.stop()
    st, site = M.moe_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error {M.moe_status_string(st)} at site {site}")
    stage_ms = {n: float(np.mean([evs[i][j].elapsed_time(evs[i][j + 1])
                                  for i in range(args.steps)]))
                for j, n in enumerate(names)}

    # end to end through the public call with host buffers
    x_h = torch.empty_like(d["x"], device="cpu").pin_memory()
    x_h.copy_(d["x"])
    l_h = torch.empty_like(d["logits"], device="cpu").pin_memory()
    l_h.copy_(d["logits"])
    xs_h = None
    if d["x_scales"] is not None:
        xs_h = torch.empty_like(d["x_scales"], device="cpu").pin_memory()
        xs_h.copy_(d["x_scales"])
    out_h = [torch.empty((T, H), dtype=ydt, device="cpu").pin_memory() for _ in range(2)]
    # two sets of device buffers, so that step i+1's inputs land and step i-1's output
    # leaves while step i computes: host->device, compute and device->host each on a stream
    x_d = [torch.empty_like(d["x"]) for _ in range(2)]
    l_d = [torch.empty_like(d["logits"]) for _ in range(2)]
    xs_d = [torch.empty_like(d["x_scales"]) if xs_h is not None else None for _ in range(2)]
    out_d = [torch.empty_like(out) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):  # every buffer starts free
        ev_comp[b].record(stream)
        ev_out[b].record(stream)

    def e2e_step(i):
        b = i % 2
        s_in.wait_event(ev_comp[b])           # step i-2 has finished reading these inputs
        with torch.cuda.stream(s_in):
            x_d[b].copy_(x_h, non_blocking=True)
            l_d[b].copy_(l_h, non_blocking=True)
            if xs_h is not None:
                xs_d[b].copy_(xs_h, non_blocking=True)
        ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])          # step i-2's output has left this buffer
        M.moe_forward(x_d[b], l_d[b], W, k, wl.score, bias=d["bias"], renorm=wl.renorm,
                      x_scales=xs_d[b], out=out_d[b], ws=fws, stream=stream)
        ev_comp[b].record(stream)
        s_out.wait_event(ev_comp[b])
        with torch.cuda.stream(s_out):
            out_h[b].copy_(out_d[b], non_blocking=True)
        ev_out[b].record(s_out)

    for i in range(args.warmup):
        e2e_step(i)
    n_e2e = max(3, min(args.steps, 20))
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    t0.record(s_in)
    for i in range(n_e2e):
        e2e_step(i)
    t1.record(s_out)
    torch.cuda.synchronize()
    barrier(ws)
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), ws) / n_e2e
    assert torch.equal(out_h[(n_e2e - 1) % 2], out_d[(n_e2e - 1) % 2].cpu())
    h2d = x_h.numel() * x_h.element_size() + l_h.numel() * 4 + (
        xs_h.numel() * 4 if xs_h is not None else 0)
    d2h = out_h[0].numel() * out_h[0].element_size()

    # roofline of the dominant kernel
    pk, pk_kind = peaks()
    alg = algorithmic(wl, touched)
    dom = max(names, key=lambda n: stage_ms[n])
    dsec = stage_ms[dom] / 1e3
    tens_mult = 2.0 if wl.act == "e4m3" else (1.0 if wl.act == "bf16" else None)
    t_flops = (alg[dom]["flops"] / (pk["bf16_tflops"] * tens_mult * 1e12)
               if (alg[dom]["flops"] and tens_mult) else 0.0)
    t_bytes = alg[dom]["bytes"] / (pk["hbm_gbs"] * 1e9)
    if t_flops >= t_bytes and alg[dom]["flops"]:
        # the kernel is timed per launch (CUDA events around one launch, a few ms inside a
        # short loop), so the burst figure is the matching peak; the power-capped sustained
        # figure, for a kernel timed inside a seconds-long loop, is reported beside it
        roof = {"bound": "tensor", "achieved": alg[dom]["flops"] / dsec / 1e12,
                "peak": pk["bf16_tflops"] * tens_mult, "unit": "TFLOP/s"}
        roof["peak_note"] = (f"{pk_kind} bf16 burst x {tens_mult:g} "
                             f"(nominal {'fp8' if tens_mult == 2 else 'bf16'}:bf16 ratio)")
        if "bf16_tflops_sustained" in pk:
            roof["frac_sustained"] = roof["achieved"] / (pk["bf16_tflops_sustained"] * tens_mult)
    else:
        roof = {"bound": "hbm", "achieved": alg[dom]["bytes"] / dsec / 1e9,
                "peak": pk["hbm_gbs"], "unit": "GB/s", "peak_note": f"{pk_kind} copy bandwidth"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dom
    if args.traffic is not None:
        roof["traffic"] = args.traffic
    elif (wl.name, dom) in TRAFFIC_RATIO and args.scale_fmt == "pow2" and args.tiles == "auto":
        # (the ratios were measured on the power-of-two-scale kernels at the automatic tile
        # shape; other paths run other kernels)
        ratio, src = TRAFFIC_RATIO[(wl.name, dom)]
        roof["traffic"] = ratio * alg[dom]["bytes"]
        roof["traffic_note"] = (f"DRAM read+write bytes per launch = {ratio} x algorithmic, "
                                f"the ratio ncu measured on {src}")
    else:
        roof["traffic"] = None
    roof["algorithmic_per_launch"] = {"bytes": alg[dom]["bytes"], "flops": alg[dom]["flops"]}

    res = {
        "metric": "fused MoE layer tokens/s (1 B200 per replica)",
        "value": T * ws / (ms / 1e3),
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"e4m3": "e4m3" if wl.wt == "e4m3" else "e4m3xe2m1", "bf16": "bf16",
                  "f32": "f32"}[wl.act],
        "data": "synthetic (seeded; random-init weights of the workload's shape)",
        "config": {"workload": wl.name, "T": T, "H": H, "E": E, "k": k, "I": I, "act": wl.act,
                   "wt": wl.wt, "router": wl.score, "experts_touched": touched,
                   "input": ("bf16, quantised to e4m3 in the dispatch" if args.bf16_input
                             else wl.act),
                   "l2": "inputs larger than L2 (expert weights >> 126 MB), no flush",
                   "parallelism": f"replicas x{ws}"},
        "tflops": wl.flops() / (ms / 1e3) / 1e12 * ws,
        "step": ("moe_forward (one persistent launch per step)" if args.scale_fmt == "pow2"
                 else "moe_forward (fp32 block scales: the chain of entry points, 9 launches)"),
        "scale_fmt": args.scale_fmt,
        "chain_ms_per_step": chain_ms,
        "stage_ms": stage_ms,
        # algorithmic bytes of each stage over its CUDA-event time, and that over the
        # measured copy bandwidth (the memory-bound stages' roofline)
        "stage_gbps": {n: alg[n]["bytes"] / (stage_ms[n] / 1e3) / 1e9 for n in names},
        "stage_hbm_frac": {n: alg[n]["bytes"] / (stage_ms[n] / 1e3) / 1e9 / pk["hbm_gbs"]
                           for n in names},
        "roofline": roof,
        "e2e": {"value": T * ws / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms, "path": "moe_forward with pinned host in/out; the copies of steps i+1 and i-1 "
                         "overlap step i's compute (three streams, two device buffer sets)"},
        "gpu_launches": int(launches),
        "gpu_launches_note": "library kernel launches in the headline timed region (one "
                             "persistent kernel per step; the per-stage breakdown loop "
                             "runs the chain of entry points, 9 launches per step)",
        "clocks": clk,
    }
    if ws == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, d, args.cpu_tokens)
    return res


def run_backward(args, ws, rank, local):
    """The BF16 layer's backward (moe_expert_backward: combine and router backward, the
    recomputed pre-activations, dh, SwiGLU backward, dx and both weight gradients) from the
    forward's stored tensors, timed per call with CUDA events."""
    import moe_expert_layer_prefix_b200 as M

    wl = workload(args)
    if wl.act != "bf16" or wl.wt != "bf16":
        raise SystemExit("--backward runs the BF16 layer (e.g. --workload mixtral_bf16)")
    dev = torch.device("cuda", torch.cuda.current_device())
    d = synth.make_inputs(wl, dev)
    W = M.Weights(wl.act, wl.wt, d["w1"], d["w2"], d["w1_scales"], d["w2_scales"])
    T, H, E, k, I, S = wl.T, wl.H, wl.E, wl.k, wl.I, wl.S
    idx, gw = M.moe_route(d["logits"], k, wl.score, bias=d["bias"], renorm=wl.renorm)
    r = M.moe_dispatch(d["x"], idx, E, wl.act)
    h, _ = M.moe_expert_linear1(r["x_perm"], r["expert_offsets"], W)
    y = M.moe_expert_linear2(h, r["expert_offsets"], W)
    w1_t, w2_t = M.moe_transpose_experts(W.w1), M.moe_transpose_experts(W.w2)
    g = torch.Generator(device=dev).manual_seed(99)
    dout = (torch.randn((T, H), generator=g, device=dev) / 64).to(torch.bfloat16)
    bws = M.workspace(M.moe_workspace_size("backward", T, H, E, k, I, "bf16", "bf16"), dev)

    def step():
        return M.moe_expert_backward(dout, d["logits"], idx, gw, r["expert_offsets"], r["slot_of"],
                                     r["x_perm"], h, y, W, w1_t, w2_t, k, score=wl.score,
                                     renorm=wl.renorm, ws=bws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, site = M.moe_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error {M.moe_status_string(st)} at site {site}")
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier(ws)
    torch.cuda.synchronize()
    n0 = M.moe_launch_count()
    for i in range(args.steps):
        evs[i].record(stream)
        step()
    evs[-1].record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    launches = M.moe_launch_count() - n0
    clk = clocks.stop()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    ms = max_over_ranks(float(np.sum(per)), ws) / args.steps
    # algorithmic FLOPs of the backward's GEMMs per step: G recomputed 4SHI, dh 2SHI,
    # dx_slot 4SHI, dW1 4SHI, dW2 2SHI
    flops = 16.0 * S * H * I
    pk, pk_kind = peaks()
    ach = flops / (ms / 1e3) / 1e12
    roof = {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
            "frac": ach / pk["bf16_tflops"], "traffic": None, "kernel": "moe_expert_backward (whole call)",
            "peak_note": f"{pk_kind} bf16 burst; the call's five GEMMs against the whole call's time"}
    return {
        "metric": "MoE layer backward tokens/s (1 B200 per replica)",
        "value": T * ws / (ms / 1e3), "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)",
        "config": {"workload": wl.name, "T": T, "H": H, "E": E, "k": k, "I": I,
                   "l2": "inputs larger than L2 (weights >> 126 MB), no flush",
                   "parallelism": f"replicas x{ws}"},
        "tflops": ach, "step": "moe_expert_backward", "roofline": roof,
        "gpu_launches": int(launches), "clocks": clk,
    }


def _oracle_layer(wl, d):
    from tests.util import oracle_layer
    return oracle_layer(wl, d, lazy_weights=True)


def _prefetch(L, wl, toks):
    import oracle
    idx, _ = oracle.route(L.logits[toks], L.bias, wl.k, wl.score, wl.renorm)
    for e in np.unique(idx):
        for arr in (L.w1, L.w2, L.w1_scales, L.w2_scales):
            if arr is not None:
                arr[e]


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(wl, d, ntok):
    """The oracle as it stands, on ntok sampled tokens of the same inputs."""
    import oracle
    L = _oracle_layer(wl, d)
    toks = np.random.default_rng(123).choice(wl.T, ntok, replace=False)
    _prefetch(L, wl, toks)
    t = time.perf_counter()
    oracle.forward_tokens(L, toks)
    dt = time.perf_counter() - t
    return {"value": ntok / dt, "unit": "tokens/s", "cores": _threads(), "kind": "oracle",
            "sample": f"{ntok} of {wl.T} tokens of {wl.name} (oracle.forward_tokens, fp64)",
            "seconds": dt}


def run_reference(args, ws, rank):
    import oracle
    wl = workload(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    d = synth.make_inputs(wl, dev)          # input generation only; the oracle runs on host
    L = _oracle_layer(wl, d)
    rng = np.random.default_rng(7)
    samples = [rng.choice(wl.T, args.ref_tokens, replace=False)
               for _ in range(args.warmup + args.steps)]
    for s in samples:
        _prefetch(L, wl, s)
    for s in samples[:args.warmup]:
        oracle.forward_tokens(L, s)
    t = time.perf_counter()
    for s in samples[args.warmup:]:
        oracle.forward_tokens(L, s)
    dt = time.perf_counter() - t
    ntok = args.ref_tokens * args.steps
    val = ntok / dt
    sample = (f"{args.ref_tokens} tokens per step of {wl.name} "
              f"(oracle.forward_tokens, fp64, host CPU)")
    return {
        "metric": "fused MoE layer tokens/s (1 B200 per replica)", "value": val,
        "unit": "tokens/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I},
        "impl": "reference",
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": _threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_route(args, ws, rank, local):
    """The router alone on the workload's logits (profiling captures of route_kernel at the
    full token count without the expert weights on the device)."""
    import moe_expert_layer_prefix_b200 as M

    wl = workload(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    d = synth.make_activations(wl, dev)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device=dev)
    gw = torch.empty((wl.T, wl.k), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        M.moe_route(d["logits"], wl.k, wl.score, bias=d["bias"], renorm=wl.renorm,
                    topk_idx=idx, topk_w=gw, stream=stream)

    for _ in range(args.warmup):
        step()
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    ms = max_over_ranks(t0.elapsed_time(t1), ws) / args.steps
    clk = clocks.stop()
    st, site = M.moe_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error {M.moe_status_string(st)} at site {site}")
    pk, pk_kind = peaks()
    byt = algorithmic(wl, wl.E)["route"]["bytes"]
    return {
        "metric": "router tokens/s (moe_route alone)", "value": wl.T * ws / (ms / 1e3),
        "unit": "tokens/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic (seeded)",
        "config": {"workload": wl.name, "T": wl.T, "E": wl.E, "k": wl.k,
                   "router": wl.score, "logits": wl.logits},
        "roofline": {"bound": "hbm", "achieved": byt / (ms / 1e3) / 1e9, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": byt / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
                     "peak_note": f"{pk_kind} copy bandwidth", "kernel": "route"},
        "clocks": clk,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="v3_fp8", choices=list(synth.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--bf16-input", action="store_true",
                    help="E4M3 workloads: feed BF16 activations, quantised in the dispatch")
    ap.add_argument("--route-only", action="store_true",
                    help="time the router alone on the workload's logits")
    ap.add_argument("--backward", action="store_true",
                    help="time the BF16 layer's backward (moe_expert_backward) instead")
    ap.add_argument("--scale-fmt", default="pow2", choices=["pow2", "fp32"],
                    help="E4M3 layers: power-of-two block scales (UE8M0 tensor-core path) or "
                         "arbitrary fp32 block scales (per-block promotion)")
    ap.add_argument("--tiles", default="auto", choices=["auto", "single", "pair", "small"],
                    help="tile shape of the expert GEMMs")
    ap.add_argument("--T", type=int, default=None, help="override T (profiling captures)")
    ap.add_argument("--E", type=int, default=None, help="override E (profiling captures)")
    ap.add_argument("--cpu-tokens", type=int, default=3)
    ap.add_argument("--ref-tokens", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel from an ncu capture")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    ws, rank, local = dist_setup(args)
    if args.impl == "reference":
        res = run_reference(args, ws, rank) if rank == 0 else None
    elif args.route_only:
        res = run_route(args, ws, rank, local)
    elif args.backward:
        res = run_backward(args, ws, rank, local)
    else:
        res = run_native(args, ws, rank, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if ws > 1 and args.impl == "native":
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
