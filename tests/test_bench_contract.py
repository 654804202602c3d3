"""bench.py's command-line contract, host only: the reference arm (the oracle
timed on the host cores) prints one JSON line with the keys and relations the
line must carry, only rank 0 prints under a multi-rank launch, and the
product arm refuses to run without a CUDA device instead of falling back to
the CPU."""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, env=None):
    e = dict(os.environ)
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        e.pop(k, None)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          env=e, capture_output=True, text=True, timeout=240)


def test_reference_arm_line():
    p = _bench("--impl", "reference", "--workload", "tiny_fp32", "--steps", "3", "--warmup", "3")
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["value"] > 0 and d["config"]["workload"] == "tiny_fp32"
    # ms_per_step is the time of one step: every branch token of the batch once
    bt = d["config"]["branch_tokens"]
    assert d["ms_per_step"] == pytest.approx(1000.0 * bt / d["value"], rel=1e-9)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["unit"] == d["unit"]
    assert cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_stay_silent():
    p = _bench("--impl", "reference", "--workload", "tiny_fp32", "--steps", "3", "--warmup", "3",
               env={"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert p.returncode == 0, p.stderr[-2000:]
    assert not [ln for ln in p.stdout.splitlines() if ln.startswith("{")]


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the refusal without a device")
def test_product_arm_needs_a_device():
    p = _bench("--workload", "tiny_fp32", "--steps", "3", "--warmup", "3")
    assert p.returncode != 0
    assert "CUDA device" in (p.stdout + p.stderr)
    assert not [ln for ln in p.stdout.splitlines() if ln.startswith("{")]


def test_bad_step_counts_are_refused():
    p = _bench("--impl", "reference", "--workload", "tiny_fp32", "--steps", "0", "--warmup", "3")
    assert p.returncode == 2 and "--steps" in p.stderr
