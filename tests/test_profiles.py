"""Host-only consistency checks of the committed profile summaries: the
attention kernel's DRAM traffic record that bench.py reports is well formed
and close to the algorithmic bytes it is compared with, and the profiles
index lists every summary."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from permuted_block_sparse_b200 import synth  # noqa: E402

PROFILES = os.path.join(ROOT, "profiles")


def test_traffic_record_is_consistent():
    with open(os.path.join(PROFILES, "attn_fwd_traffic.json")) as f:
        j = json.load(f)
    w = synth.WORKLOADS[j["workload"]]
    assert len(j["attn_fwd_sha"]) == 16 and int(j["attn_fwd_sha"], 16) >= 0
    assert j["bytes_per_launch"] == j["dram_bytes_read"] + j["dram_bytes_write"]
    # Q, K, V and O once (bf16) plus LSE (fp32): the algorithmic minimum
    algorithmic = (2 * w.B * w.Hq * w.N * w.d * 2 + 2 * w.B * w.Hkv * w.N * w.d * 2 + w.B * w.Hq * w.N * 4)
    assert 0.85 * algorithmic <= j["bytes_per_launch"] <= 1.10 * algorithmic
    assert "--clock-control none" in j["command"] and "-k regex:attn_fwd" in j["command"]


def test_profiles_index_lists_every_summary():
    with open(os.path.join(PROFILES, "README.md")) as f:
        index = f.read()
    for name in os.listdir(PROFILES):
        if name != "README.md":
            assert f"`{name}`" in index, name
        assert not name.endswith((".ncu-rep", ".nsys-rep", ".qdrep")), name
