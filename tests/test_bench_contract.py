"""The bench's JSON line, checked on the CPU: the reference arm (the oracle on a
bounded sample) prints one line with every key the contract names, and the
product arm refuses to run without a GPU instead of falling back to the CPU."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
             "scaling", "vs_baseline", "dtype", "data", "config"}


def _bench(*args, timeout=300):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, env=env, capture_output=True,
                          text=True, timeout=timeout)


@pytest.mark.parametrize("args, unit", [
    (["--config", "1"], "GB/s"),
    (["--workload", "prefill", "--prefill-workload", "prefill-tiny"], "TFLOP/s"),
])
def test_reference_arm_prints_one_complete_line(args, unit):
    r = _bench("--impl", "reference", *args, "--steps", "2", "--warmup", "3", "--ref-step-budget", "0.2")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert BASE_KEYS <= set(d)
    assert d["impl"] == "reference" and d["unit"] == unit
    assert d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["vs_baseline"] is None and d["data"] == "synthetic" and d["dtype"] == "f64"
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == unit
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_product_arm_needs_a_gpu():
    r = _bench("--steps", "3", "--warmup", "3", "--no-cpu-baseline", timeout=120)
    assert r.returncode != 0
    assert not [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_more_than_one_gpu_needs_torchrun():
    r = _bench("--gpus", "2", "--steps", "3", "--warmup", "3", timeout=120)
    assert r.returncode != 0
    assert "torchrun" in r.stderr
