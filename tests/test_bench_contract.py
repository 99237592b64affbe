"""The benchmark's reference arm (the fp64 oracle timed on the host cores)
prints the contract's JSON line; it needs no GPU, so it is checked here."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_reference_arm_prints_the_contract_line():
    line = _run("--impl", "reference", "--steps", "2", "--warmup", "3", "--ref-seconds", "2")
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["steps"] == 2 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["config"]["workload"] == "nsa_decode_bf16_b32_l65536"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_on_a_prefill_workload():
    line = _run("--impl", "reference", "--workload", "nsa_prefill_bf16_t8192", "--steps", "1",
                "--warmup", "3", "--ref-seconds", "2")
    assert line["unit"] == "TFLOP/s" and line["value"] > 0


def test_reference_arm_on_the_moba_workload():
    line = _run("--impl", "reference", "--workload", "moba_prefill_bf16_t131072", "--steps", "1",
                "--warmup", "3", "--ref-seconds", "2")
    assert line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["config"]["workload"] == "moba_prefill_bf16_t131072"
