"""bench.py's reference arm on the CPU: the float64 oracle timed on the host cores.

The arm runs without a GPU, so its JSON line (the keys the benchmark contract fixes) and its behaviour
under torchrun (rank 0 alone prints; the other ranks exit 0 without work) are checked here.
"""
from __future__ import annotations

import json
import os
import subprocess
import sys

import bench
from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env: dict, *args: str) -> subprocess.CompletedProcess:
    env = dict(os.environ)
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        env.pop(k, None)
    env.update(extra_env)
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=300)


def test_reference_arm_prints_one_contract_line():
    r = _run({}, "--steps", "2", "--warmup", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["vs_baseline"] is None and d["data"] == "synthetic" and d["scaling"] in ("weak", "strong")
    # one step: one (batch, head) unit of the default workload's tokens
    wl = WORKLOADS["pvt1"]
    assert abs(d["value"] * d["ms_per_step"] * 1e-3 - wl.N) <= 1e-6 * wl.N
    assert d["config"]["workload"] == bench.workload_config(wl, {})["workload"]
    assert d["config"]["whiten"] == "unit"   # the default arm's column statistics, per (batch, head) unit
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    r = _run({"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"}, "--gpus", "2", "--steps", "1", "--warmup", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]
