"""bench.py's reference arm (the float64 oracle on the host cores) keeps the
JSON-line contract the GPU arm keeps, on CPU: one line on rank 0, nothing on
the other ranks, and an `unavailable` line for workloads it does not time."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         capture_output=True, text=True, cwd=ROOT, env=env, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    return [ln for ln in out.stdout.splitlines() if ln.strip()]


def test_reference_arm_line():
    lines = _run("--impl", "reference", "--workload", "1", "--steps", "2", "--warmup", "1")
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for k in ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"]:
        assert k in d, k
    assert d["value"] > 0 and d["unit"] == "EM iters/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] and d["data"] == "synthetic"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_print_nothing():
    assert _run("--impl", "reference", "--workload", "1", "--steps", "1", "--warmup", "1",
                env_extra={"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_reference_arm_kmeans_is_unavailable():
    lines = _run("--impl", "reference", "--workload", "4", "--steps", "1", "--warmup", "1")
    d = json.loads(lines[-1])
    assert d["impl"] == "reference" and d["unavailable"]
