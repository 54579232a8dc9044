"""The benchmark's output contract and the absence of any CPU fallback, checked
without a GPU: the reference arm (the fp64 oracle timed on the host cores)
prints one JSON line with the contract's keys; the native arm and the binding
fail loudly when there is no GPU or no library."""
import json
import os
import subprocess
import sys

import pytest
import torch

from sparse_linear_attention_mean_b200 import binding as rb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=300):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["value"] > 0 and j["ms_per_step"] > 0 and j["steps"] == 1
    assert j["config"]["workload"] == "wan14b-720p-s97"
    assert j["config"]["k_b"] == 18 and j["config"]["n_blocks"] == 591
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == j["value"]
    assert j["e2e"] == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_native_arm_fails_without_a_gpu():
    r = _run("--steps", "1", "--warmup", "1", "--no-cpu-baseline")
    assert r.returncode != 0
    assert not any(ln.startswith("{") for ln in r.stdout.splitlines())


def test_binding_raises_when_the_library_is_missing(monkeypatch):
    monkeypatch.setattr(rb, "_lib", None)
    monkeypatch.setattr(rb, "LIB_PATH", os.path.join(ROOT, "no-such-dir", "librola.so"))
    with pytest.raises(RuntimeError, match="missing"):
        rb.lib()
