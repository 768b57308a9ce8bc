"""The benchmark's output contract on the CPU: the reference arm (the oracle) and the
admission-scheduler mode print one JSON line with the keys and types the driver reads."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    d = run_bench("--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3")
    assert d["impl"] == "reference"
    for key, typ in [("metric", str), ("value", float), ("unit", str), ("n_gpus", int), ("steps", int),
                     ("warmup", int), ("ms_per_step", float), ("higher_is_better", bool), ("scaling", str),
                     ("dtype", str), ("data", str), ("config", dict), ("cpu_baseline", dict), ("e2e", dict)]:
        assert isinstance(d[key], typ), key
    assert d["steps"] == 2 and d["warmup"] == 3 and d["value"] > 0
    assert d["vs_baseline"] is None and "workload" in d["config"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1


def test_warmup_below_three_is_refused():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert out.returncode != 0


def test_scheduler_mode_line():
    d = run_bench("--sched")
    assert d["unit"] == "pages/1k tokens" and d["higher_is_better"] is False and d["n_gpus"] == 1
    runs = d["runs"]
    assert set(runs) == {"aimd", "fixed256_offload", "fixed256_recompute"}
    assert all(r["done"] == 512 and r["stalled"] == 0 for r in runs.values())
    assert d["value"] == runs["aimd"]["pages_per_1k_tokens"]
    # the model's headline: AIMD moves far fewer pages than a fixed cap of 256 with offload
    assert runs["aimd"]["pages_per_1k_tokens"] < 0.5 * runs["fixed256_offload"]["pages_per_1k_tokens"]
    assert runs["fixed256_recompute"]["pages_per_1k_tokens"] == 0.0
    assert d["cpu_baseline"]["kind"] == "oracle"
