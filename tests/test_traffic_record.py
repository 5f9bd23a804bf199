"""The attention kernel's recorded DRAM traffic (profiles/*.traffic.json)
stays usable while only host code changes: the record carries a SHA-256 over
the kernel's device sources alone and one over everything the bench hashes
(device sources plus the host file that launches the kernel). If the device
sources are unchanged the full hash must match too, i.e. the record was
re-stamped after the host-only edit; if they changed, the counters are stale
and the bench reports traffic as null, which this test accepts. CPU only."""
import hashlib
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "transformer_attention_gqa_b200", "csrc")


def _sha(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(CSRC, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def test_recorded_traffic_is_restamped_after_host_only_edits():
    path = os.path.join(ROOT, "profiles", "gqa_attn_fwd_kernel.llama8b.traffic.json")
    with open(path) as f:
        rec = json.load(f)
    assert set(rec["device_sources"]) <= set(bench.KERNEL_SOURCES)
    if _sha(rec["device_sources"]) == rec["device_sources_sha256"]:
        assert bench.recorded_traffic("llama8b") == int(rec["dram_bytes_per_launch"]), \
            "kernel unchanged but the record's full hash is stale: re-stamp sources_sha256"
    else:
        assert bench.recorded_traffic("llama8b") is None
