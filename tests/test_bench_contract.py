"""The bench's host side on CPU: the algorithmic work it divides by (the roofline's
numerator) against a brute-force count from the attention's definition, and the
JSON line of the reference arm (the oracle timed on host cores) against the
contract's keys."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import bench
from gqa_attention_forward_flash_b200.synth import WORKLOADS, Workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _brute_force(w: Workload, lens):
    """Visible (query row, key) pairs and visible key rows, by enumeration: row i of a
    head sees key j iff j < n and (not causal or j <= n - Tq + i)."""
    pairs = 0
    kv_rows = 0
    for n in lens:
        seen = np.zeros(max(n, 1), bool)
        for i in range(w.Tq):
            for j in range(n):
                if (not w.causal) or j <= n - w.Tq + i:
                    pairs += 1
                    seen[j] = True
        kv_rows += int(seen[:n].sum())
    # per KV head: every one of its G query heads sees the same pairs; K and V rows once
    flops = 4 * w.d * pairs * w.G * w.Hkv
    nbytes = (2 * kv_rows * w.d * 2) * w.Hkv + len(lens) * w.Hkv * (2 * w.G * w.Tq * w.d * 2 + w.G * w.Tq * 4)
    return nbytes, flops


@pytest.mark.parametrize("w,lens", [
    (Workload("a", B=3, Hq=8, Hkv=2, Tq=5, Tkv=40, d=64, causal=True), [40, 3, 0]),
    (Workload("b", B=2, Hq=4, Hkv=4, Tq=7, Tkv=30, d=128), [30, 11]),
    (Workload("c", B=2, Hq=6, Hkv=2, Tq=1, Tkv=50, d=64, causal=True), [50, 1]),
])
def test_algorithmic_work_matches_enumeration(w, lens):
    assert bench.workload_work(w, lens) == _brute_force(w, lens)


def test_full_causal_prefill_flops_closed_form():
    w = WORKLOADS["full_causal_prefill"]
    _, flops = bench.workload_work(w, None)
    # every row i sees i + 1 keys: 4·d·Σ(i+1) per head
    assert flops == 4 * w.B * w.Hq * w.d * (w.Tq * (w.Tq + 1) // 2)


def test_reference_arm_line_keeps_the_contract():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                        "--ref-step-seconds", "0.3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["warmup"] >= 3 and line["steps"] == 1 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["config"]["workload"] == "batched_decode"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
