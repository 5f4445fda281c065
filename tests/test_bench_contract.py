"""bench.py's command-line contract, checked on the host: the reference arm (the oracle timed
on the CPU) prints one JSON line with the required keys, and too few warm-up steps are
rejected."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
        "cpu_baseline", "e2e")


def _bench(*args, timeout=600):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=timeout, cwd=ROOT)


def test_reference_arm_prints_the_json_line():
    r = _bench("--impl", "reference", "--workload", "tiny_f32", "--steps", "3", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    for key in KEYS:
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["config"]["workload"] == "tiny_f32"
    assert d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_too_few_warmup_steps_are_rejected():
    r = _bench("--impl", "reference", "--workload", "tiny_f32", "--steps", "3", "--warmup", "2",
               timeout=120)
    assert r.returncode != 0
    assert "warmup" in r.stderr


def test_algorithmic_units_match_the_published_workload_figures():
    """The roofline's algorithmic FLOPs and weight bytes against figures computed by hand: the
    two GEMMs are 6 S H I FLOP (V3 5.772 TFLOP, Mixtral 2.886 TFLOP, decode 90.2 GFLOP); all
    experts' weights are 11.27 GB for V3 (E4M3 codes + fp32 128x128 scales) and 2.82 GB for
    Mixtral (BF16)."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    for name, tflop in (("v3_fp8", 5.772), ("mixtral_bf16", 2.886), ("decode_fp8_fp4", 0.0902)):
        wl = synth.WORKLOADS[name]
        a = bench.algorithmic(wl, wl.E)
        total = a["linear1"]["flops"] + a["linear2"]["flops"]
        assert abs(total / 1e12 - tflop) / tflop < 5e-4, (name, total)
    v3 = synth.WORKLOADS["v3_fp8"]
    a = bench.algorithmic(v3, v3.E)
    act = v3.S * (v3.H + v3.H // 128 * 4) + v3.S * (v3.I + v3.I // 128 * 4)
    weights = a["linear1"]["bytes"] - act + (a["linear2"]["bytes"] - v3.S * (v3.I + v3.I // 128 * 4)
                                             - v3.S * v3.H * 2)
    assert abs(weights / 1e9 - 11.27) < 0.01, weights
    mx = synth.WORKLOADS["mixtral_bf16"]
    a = bench.algorithmic(mx, mx.E)
    weights = (a["linear1"]["bytes"] - mx.S * (mx.H + mx.I) * 2 +
               a["linear2"]["bytes"] - mx.S * mx.I * 2 - mx.S * mx.H * 2)
    assert abs(weights / 1e9 - 2.82) < 0.01, weights


def test_algorithmic_bytes_of_the_decode_weights_and_the_router():
    """The byte counts behind the HBM rooflines, against hand-computed figures: the decode
    layer's E2M1 weights with their UE8M0 per-32 scales are 3 x I x H x (1/2 + 1/32) bytes
    per expert (23.4 MB; 5.89 GB for the 252 experts its routing touches), and the router
    reads T x E fp32 logits and writes T x k indices and gates (69.2 MB on the skewed
    layer)."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    wl = synth.WORKLOADS["decode_fp8_fp4"]
    per_expert = 3 * wl.I * wl.H * (0.5 + 1 / 32)
    assert abs(per_expert / 1e6 - 23.4) < 0.05
    a = bench.algorithmic(wl, 252)
    act = wl.S * (wl.H + wl.H // 128 * 4) + 2 * wl.S * (wl.I + wl.I // 128 * 4) + wl.S * wl.H * 2
    weights = a["linear1"]["bytes"] + a["linear2"]["bytes"] - act
    assert abs(weights / 1e9 - 5.89) < 0.01, weights
    sk = synth.WORKLOADS["skewed_fp8_fp4"]
    assert bench.algorithmic(sk, sk.E)["route"]["bytes"] == sk.T * sk.E * 4 + sk.T * sk.k * 8
    assert abs(bench.algorithmic(sk, sk.E)["route"]["bytes"] / 1e6 - 69.2) < 0.1
