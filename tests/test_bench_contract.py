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
