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


@pytest.mark.parametrize("workload", ["tiny", "decode_small", "bwd_nano", "qkv_nano", "masked_nano", "rot_nano"])
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
    assert res["config"] == json.loads(json.dumps(_gpu_arm_config(workload)))  # the GPU arm's config, key for key
    assert res["cpu_baseline"]["kind"] == "oracle" and res["cpu_baseline"]["cores"] >= 1
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["e2e"]["d2h_bytes_per_step"] == 0


def _gpu_arm_config(workload):
    sys.path.insert(0, ROOT)
    import bench
    from transformer_attention_gqa_b200 import workloads as wl

    if workload in wl.DECODE_WORKLOADS:
        return bench.decode_config(wl.DECODE_WORKLOADS[workload], 1)
    if workload in bench.BWD_WORKLOADS:
        w = wl.WORKLOADS[bench.BWD_WORKLOADS[workload]]
        return bench.bwd_config(workload, w, 1, bench.BWD_FLOP_FACTOR * w.flops())
    if workload in bench.PROJ_WORKLOADS:
        return bench.proj_config(workload, wl.WORKLOADS[bench.PROJ_WORKLOADS[workload]], 1)
    if workload in bench.MASKED_WORKLOADS:
        w = wl.WORKLOADS[bench.MASKED_WORKLOADS[workload]]
        return bench.masked_config(workload, w, 1, bench._bench_mask(w, w.seed + 1).shape)
    if workload in bench.ROT_WORKLOADS:
        return bench.fwd_config(wl.WORKLOADS[bench.ROT_WORKLOADS[workload]], 1, workload)
    return bench.fwd_config(wl.WORKLOADS[workload], 1)


def test_forward_roofline_picks_the_binding_unit():
    """Long sequences at d = 128 are bound by the tensor cores; at d = 64 the
    exponentials (one per visible pair and head, on the special-function
    unit) take longer than the products."""
    sys.path.insert(0, ROOT)
    import bench
    from transformer_attention_gqa_b200 import workloads as wl

    peaks = {"bf16_tflops": 1628.3, "hbm_gbs": 6535.0}
    clk = {"sm_mhz": 1965.0}
    llama = bench.fwd_roofline(wl.WORKLOADS["llama8b"], 0.5, peaks, "measured", clk, 148)
    assert llama["bound"] == "tensor" and llama["unit"] == "TFLOP/s"
    assert abs(llama["achieved"] - wl.WORKLOADS["llama8b"].flops() / 0.5e-3 / 1e12) < 0.01
    qwen = bench.fwd_roofline(wl.WORKLOADS["qwen05b"], 0.08, peaks, "measured", clk, 148)
    assert qwen["bound"] == "alu" and qwen["unit"] == "Gexp/s"
    assert abs(qwen["peak"] - 16 * 148 * 1.965) < 0.1
    assert set(qwen["others"]) == {"tensor", "hbm"}
