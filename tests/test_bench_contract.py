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


def test_mismatched_world_size_is_refused():
    # a launcher that started one rank while the command asks for two must not print a 1-GPU line
    r = _bench("--gpus", "2", "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3",
               timeout=120)
    assert r.returncode == 2 and "WORLD_SIZE=1" in r.stderr and not r.stdout.strip()


def test_gpus_without_launcher_spawns_ranks():
    # no WORLD_SIZE in the environment: bench.py starts its own two ranks (rank 0 prints the line)
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "3"], cwd=ROOT, capture_output=True,
                       text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"


def test_peak_choice_follows_region_length_and_clocks():
    import bench
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    capped = {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.tensor_peak(peaks, "measured", capped, 0.2)[0] == 1600.0     # short region: burst
    assert bench.tensor_peak(peaks, "measured", full, 5.0)[0] == 1600.0       # long but at full clock
    assert bench.tensor_peak(peaks, "measured", dict(capped, reasons=[]), 5.0)[0] == 1600.0
    p, src = bench.tensor_peak(peaks, "measured", capped, 5.0)                # long and power-capped
    assert p == 1400.0 and "sustained" in src and "1700" in src
    assert bench.tensor_peak(peaks, "fallback", None, 0.1)[1].startswith("fallback burst")
    # a launch bound by HBM reports GB/s against the copy bandwidth
    roof, _, _ = bench.tensor_or_hbm_roofline(1e9, 6.5e9, 1.0, peaks, "measured", full, 0.1)
    assert roof["bound"] == "hbm" and roof["frac"] == 1.0
    roof, _, _ = bench.tensor_or_hbm_roofline(1.6e12, 1e6, 2.0, peaks, "measured", full, 0.1)
    assert roof["bound"] == "tensor" and roof["frac"] == 0.5


def test_per_config_covers_every_configuration():
    import bench
    from spacetime_attention_b200 import synthetic as syn
    names = {n for n, _ in bench.PER_CONFIG}
    assert names == set(syn.WORKLOADS)
    for n, kind in bench.PER_CONFIG:
        assert kind == "dense" or syn.WORKLOADS[n].skiparse_k
    assert ("long_video", "skiparse") in bench.PER_CONFIG and ("long_video", "dense") in bench.PER_CONFIG
