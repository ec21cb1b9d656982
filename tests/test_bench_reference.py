"""The reference arm of bench.py (the fp64 oracle timed on host cores) on the
small workload: one JSON line with the contract's keys, the workload's
identity (admitted pairs in closed form) and the forward or backward metric."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("pass_", ["fwd", "bwd"])
def test_reference_arm_line(pass_):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny_ring_fp32",
           "--steps", "2", "--warmup", "3", "--pass", pass_]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, check=True).stdout.strip().splitlines()
    assert len(out) == 1
    d = json.loads(out[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    S = 1024
    assert d["config"]["admitted_pairs"] == S * (S + 1) // 2
    assert d["metric"].startswith("ring-attn bwd" if pass_ == "bwd" else "ring-attn fwd")
    assert d["config"]["flops_per_step"] == (10.0 if pass_ == "bwd" else 4.0) * 64 * 4 * S * (S + 1) // 2
