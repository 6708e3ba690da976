"""CPU tests of bench.py's reference arm (the oracle timed on host cores):
it runs the warm-up and timed steps, prints one JSON line with the fields the
bench contract fixes, and a non-zero rank exits 0 without work."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None, steps=1, warmup=3):
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env.update(extra_env or {})
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", str(steps),
                           "--warmup", str(warmup)], cwd=ROOT, env=env, capture_output=True,
                          text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run(steps=2)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    # the GPU arm's metric; the config names the bounded sample of its workload
    # that the oracle actually times
    w = bench.oracle_sample_workload()
    assert d["metric"] == bench.METRIC and d["config"] == bench.reference_config(w)
    assert f"B={w.B}, Hq={w.Hq}, Hkv={w.Hkv}, N={w.Nq}" in d["config"]["workload"]
    assert d["config"]["sample_of"] == bench.STEP_WORKLOAD
    # value is the FLOP rule's fwd + bwd FLOPs of the sample over the mean step time
    fwd = 4 * w.B * w.Hq * w.Nq * w.Nk * w.d / 2   # causal halves the forward
    flops = fwd * 3.5                               # bwd = 2.5 x fwd
    assert abs(flops / (d["ms_per_step"] * 1e-3) / 1e12 - d["value"]) <= 1e-9 * d["value"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(extra_env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
