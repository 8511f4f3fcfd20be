"""CPU checks of bench.py's command-line contract: the reference arm (the
oracle timed on the host cores) prints one JSON line with the contract's
keys, and the library arm refuses to run without a GPU instead of falling
back to a CPU path."""
from __future__ import annotations

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


def test_reference_arm_prints_the_contract_line():
    res = _run("--impl", "reference", "--steps", "1", "--warmup", "3")
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    out = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in out, k
    assert out["impl"] == "reference"
    assert out["value"] > 0 and out["steps"] == 1 and out["warmup"] == 3
    assert out["higher_is_better"] is True and out["vs_baseline"] is None
    assert out["config"]["workload"] == "llama7b_attn_proj_4096x4096_m4096_r16"
    cb = out["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == out["value"]
    assert cb["sample"]
    assert out["e2e"] == {"value": out["value"], "unit": out["unit"],
                          "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_warmup_below_three_is_refused():
    res = _run("--impl", "reference", "--steps", "1", "--warmup", "2")
    assert res.returncode != 0
    assert not [ln for ln in res.stdout.splitlines() if ln.startswith("{")]


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_library_arm_needs_a_gpu():
    res = _run("--steps", "3", "--warmup", "3", timeout=120)
    assert res.returncode != 0
    assert not [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
