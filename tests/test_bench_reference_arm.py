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


def test_issued_mma_flops_per_pair():
    """The issued-FLOP counts the bench line reports beside 6NKd and 8NKd,
    from the kernels' MMA programs: the cluster kernel on fp32 X issues
    12d (E-step) + 12d + 64 (M-step, S0); two sweeps on 16-bit X 10d twice +
    10d + 64; the small-mixture kernel at d = 32, K = 16: 12d + 32d."""
    sys.path.insert(0, ROOT)
    import bench
    f = bench.issued_mma_flops_per_pair
    assert f("tcgen05-single-sweep-cluster", "f32", 128, 256) == 24 * 128 + 64
    assert f("tcgen05-single-sweep-cluster", "bf16", 128, 256) == 20 * 128 + 64
    assert f("tcgen05-two-sweep", "bf16", 128, 4096) == 30 * 128 + 64
    assert f("tcgen05-single-sweep-smallk", "bf16", 32, 16) == 44 * 32
    assert f("simt-two-sweep", "f32", 16, 8) is None
