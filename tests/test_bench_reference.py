"""bench.py's reference arm (the float64 oracle timed on the host cores), run as
the driver runs it, on the tiny fp32 workload and on a bounded sample of the
LongNet-base layer: one JSON line with the contract's keys, the sample never
longer than the workload, and no GPU touched."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*extra, env_extra=None):
    env = dict(os.environ)
    env["CUDA_VISIBLE_DEVICES"] = ""
    env.update(env_extra or {})
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          *extra], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    return json.loads(lines[0])


def _check_contract(line, steps, warmup):
    assert line["impl"] == "reference"
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["steps"] == steps and line["warmup"] == warmup and line["n_gpus"] == 1
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["dtype"] == "f64" and line["data"] == "synthetic"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_tiny_sample_is_the_whole_workload():
    line = _run("--workload", "tiny_f32", "--steps", "1", "--warmup", "3")
    _check_contract(line, 1, 3)
    assert line["config"]["workload"] == "tiny_f32" and line["config"]["N"] == 512
    assert "positions [0, 512)" in line["cpu_baseline"]["sample"]


def test_reference_arm_default_workload_is_sampled():
    line = _run("--steps", "1", "--warmup", "3", "--reference-seconds", "8")
    _check_contract(line, 1, 3)
    assert line["config"]["workload"] == "longnet_base_32k"
    sample = line["cpu_baseline"]["sample"]
    n = int(sample.split("positions [0, ")[1].split(")")[0])
    assert 2048 <= n <= 32768 and n % 2048 == 0


def test_reference_arm_other_ranks_print_nothing():
    env = {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "3"], cwd=ROOT,
                         env=dict(os.environ, CUDA_VISIBLE_DEVICES="", **env),
                         capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr[-2000:]
    assert not [ln for ln in res.stdout.splitlines() if ln.startswith("{")]


def test_bench_refuses_fewer_than_three_warmup_steps():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"],
                         cwd=ROOT, capture_output=True, text=True, timeout=120,
                         env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert res.returncode == 2 and "--warmup must be at least 3" in res.stderr
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"], cwd=ROOT,
                         capture_output=True, text=True, timeout=120)
    assert res.returncode == 0 and "--impl" in res.stdout and "--reference-seconds" in res.stdout
