"""bench.py's reference arm (the fp64 oracle on the host cores) keeps the JSON
line contract: one line with the metric, the workload, the timing fields, a
cpu_baseline describing the run and an e2e object with no copies.  Runs on
the CPU on the tiny configuration; under torchrun only rank 0 prints."""

import json
import os
import subprocess
import sys

import bench
from kv_cache_eviction_scores_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None, *args):
    env = dict(os.environ, **(extra_env or {}))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--config", "0", *args], env=env, capture_output=True, text=True,
                          timeout=600, cwd=ROOT)


def test_reference_arm_line():
    out = _run(None, "--steps", "2", "--warmup", "1")
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 2, 1)
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["vs_baseline"] is None and d["data"] == "synthetic" and d["dtype"] == "f64"
    spec = W.config_spec(0)
    assert d["config"]["workload"] == bench.workload_desc(spec)
    # value is tokens per second of the whole workload: consistent with ms_per_step
    assert abs(d["value"] * d["ms_per_step"] / 1e3 - sum(spec.lengths)) <= 1e-6 * sum(spec.lengths)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["unit"] == d["unit"]
    assert cb["cores"] >= 1 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    out = _run({"RANK": "1", "WORLD_SIZE": "2"}, "--steps", "1", "--warmup", "0")
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip() == ""
