"""Host-only checks of bench.py: the reference arm (the oracle on the host
cores) prints one well-formed JSON line, and the algorithmic byte counts the
GPU arm reports follow from the workload's shapes."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from permuted_block_sparse_b200 import synth  # noqa: E402


def test_reference_arm_prints_one_json_line():
    import time
    t0 = time.perf_counter()
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "single_head_1k", "--steps", "2", "--warmup", "0"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    wall = time.perf_counter() - t0
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s"
    assert d["higher_is_better"] is True and d["value"] > 0
    assert d["config"] == bench.arm_config(synth.WORKLOADS["single_head_1k"])
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    # ms_per_step is the time a step actually ran, so the steps fit in the run's wall time;
    # the 1K workload (16 query blocks) is small enough to run in full
    assert 0 < d["ms_per_step"] * d["steps"] <= wall * 1e3
    assert "the whole workload" in d["cpu_baseline"]["sample"]
    assert d["est_full_run_s"] == pytest.approx(d["ms_per_step"] / 1e3, rel=0.5)


def test_oracle_baseline_sample_states_its_fraction():
    w = synth.WORKLOADS["gqa_8k_band"]
    Q, K, V, _ = synth.make_inputs(w)
    cpu = bench.oracle_baseline(w, Q, K, V, budget_s=2.0, n_blocks=4)
    n_rows = w.B * w.Hq * w.nb
    assert f"of {n_rows} query blocks" in cpu["sample"] and "divided by its sampled fraction" in cpu["sample"]
    assert 0 < cpu["fraction_of_attention"] <= 4 / n_rows
    assert cpu["est_full_run_s"] > cpu["sample_s"] > 0


def test_algorithmic_bytes():
    w = synth.WORKLOADS["llama8b_128k_sink"]
    k = w.B * w.Hkv * w.N * w.d * 2
    assert bench.permute_bytes(w) == k + w.B * w.Hq * w.blk * w.d * 2 + w.B * w.Hkv * w.N * 4
    q = w.B * w.Hq * w.N * w.d * 2
    pooled = w.B * w.Hq * w.nb * w.d * 4 + 2 * w.B * w.Hkv * w.nb * w.d * 4
    assert bench.select_bytes(w, 99) == q + k + 2 * pooled + w.B * w.Hq * w.nb * 100 * 4
    for name in ("gate_b1_64k", "sample_32k_local"):
        assert bench.permute_bytes(synth.WORKLOADS[name]) is None
        assert bench.select_bytes(synth.WORKLOADS[name], 1) is None
    assert bench._gbs(None, 1.0) is None and bench._gbs(2e9, 1000.0) == pytest.approx(2.0)


def test_dense_flops_and_labels():
    w = synth.WORKLOADS["llama8b_128k_sink"]
    assert bench.dense_causal_flops(w) == 2.0 * 128 * 131072 ** 2 * 32
    assert "topk density=0.1" in bench.selection_label(w) and "n_sink=128" in bench.selection_label(w)
    assert bench.selection_label(synth.WORKLOADS["sample_32k_local"]).startswith("SampleAttention-style")


def test_step_launches():
    """The kernels one bench step launches, as the library's entry points
    issue them: 2 permutation, 4 selection (one key-pooling launch per key
    permutation), 1 attention."""
    W = synth.WORKLOADS
    assert bench.step_launches(W["llama8b_128k_sink"]) == 7
    assert bench.step_launches(W["llama8b_32k_tau"]) == 7
    assert bench.step_launches(W["s2o_32k_stop"]) == 7
    w = W["s2o_32k_segperm"]
    assert bench.step_launches(w) == 6 + w.N // w.seg
    assert bench.step_launches(W["s2o_32k_qperm"]) == 10
    assert bench.step_launches(W["sample_32k_local"]) == 4
    for name in ("gate_b8_2k", "gate_b8_4k", "gate_b1_64k"):
        assert bench.step_launches(W[name]) == 1
