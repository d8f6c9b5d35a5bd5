"""The bench's reference arm (the fp64 oracle timed on the host cores) on CPU: one JSON line with
the bench's keys, and under a multi-rank launch only rank 0 runs and prints it (the other ranks
exit 0 without work). The tiny workload keeps each sample to milliseconds."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline",
        "e2e")


def _run(gpus, env_extra):
    env = dict(os.environ, **env_extra)
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "1", "--steps", "2",
           "--warmup", "3", "--gpus", str(gpus)]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r, [line for line in r.stdout.splitlines() if line.startswith("{")]


def test_reference_arm_prints_one_contract_line():
    r, lines = _run(1, {})
    assert r.returncode == 0, r.stderr[-2000:]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert all(k in d for k in KEYS), sorted(set(KEYS) - set(d))
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert (d["steps"], d["warmup"], d["n_gpus"]) == (2, 3, 1)
    assert d["higher_is_better"] is True and d["vs_baseline"] is None and d["dtype"] == "f64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_0_only():
    r, lines = _run(2, {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert lines == []
