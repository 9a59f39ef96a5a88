"""bench.py's host-side contract on CPU: the reference arm (the fp64 oracle on the host cores)
prints one JSON line with the keys the measurement contract names, and bad flag combinations
are refused before any device work."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config"}


def _bench(*args, timeout=300):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, capture_output=True,
                          text=True, timeout=timeout, env=dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0"))


def test_reference_arm_prints_one_contract_line():
    r = _bench("--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert KEYS <= set(line)
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["steps"] == 2 and line["warmup"] == 3
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["config"]["workload"] == "tiny"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


@pytest.mark.parametrize("args", [
    ["--warmup", "2"],                                   # fewer than 3 warm-up steps
    ["--attn", "spatial"],                               # a backward-only form on the forward step
    ["--op", "cross", "--attn", "temporal_causal"],
    ["--op", "nonexistent"],
])
def test_bad_flags_are_refused(args):
    r = _bench(*args, timeout=120)
    assert r.returncode == 2 and "error" in r.stderr
