"""bench.py's command-line contract on the CPU.

The reference arm (`--impl reference`) times the float64 oracle on the host cores and
prints one JSON line with the keys the launcher reads. The product arm has no CPU path:
on a machine without a GPU it exits non-zero and prints no result line."""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=300):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


def _json_lines(text):
    return [json.loads(x) for x in text.splitlines() if x.startswith("{")]


def test_reference_arm_prints_one_complete_line():
    r = _run("--impl", "reference", "--steps", "2", "--warmup", "3", "--ref-tokens", "64",
             "--ref-seconds", "0")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference"
    assert d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["metric"].startswith("KDA prefill tokens/s")
    assert d["config"]["workload"].startswith("t8k_h12")
    assert d["data"] == "synthetic" and d["scaling"] == "weak"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "64 tokens" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the machine without a GPU")
def test_product_arm_fails_loudly_without_a_gpu():
    r = _run("--steps", "1", "--warmup", "3", "--no-cpu-baseline")
    assert r.returncode != 0
    assert _json_lines(r.stdout) == []
