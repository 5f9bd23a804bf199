"""The benchmark's reference arm (the float64 oracle on host cores) prints
one JSON line with the contract's keys, for a prefill, a decoding, a
backward, a projection and a masked-attention workload. CPU only: the reference arm needs no GPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


@pytest.mark.parametrize("workload", ["tiny", "decode_small", "bwd_nano", "qkv_nano", "masked_nano"])
def test_reference_arm_json_line(workload):
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", workload,
                        "--steps", "2", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert KEYS <= set(res)
    assert res["impl"] == "reference" and res["value"] > 0 and res["steps"] == 2 and res["warmup"] == 3
    assert res["config"]["workload"] == workload
    assert res["cpu_baseline"]["kind"] == "oracle" and res["cpu_baseline"]["cores"] >= 1
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["e2e"]["d2h_bytes_per_step"] == 0
