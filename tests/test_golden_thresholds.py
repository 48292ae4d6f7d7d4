"""The stored gate thresholds are the oracle's calibration of the seeded
workload inputs ("Block Sparse Flash Attention", Approach: thresholds are
calibrated offline to keep roughly the top-k tiles).  Re-derive a sample of
them from the oracle and compare exactly; check the shape and the -inf rule
for blocks with at most `keep` causal tiles."""
import os

import numpy as np
import pytest

import oracle
from permuted_block_sparse_b200 import synth

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("name", ["gate_b8_2k", "gate_b8_4k", "gate_b1_64k"])
def test_stored_thresholds_match_oracle(name):
    w = synth.WORKLOADS[name]
    thr = np.load(os.path.join(HERE, f"gate_thr_{name}.npy"))
    assert thr.dtype == np.float32 and thr.shape == (w.B, w.Hq, w.nb)
    i = np.arange(w.nb)
    few = i + 1 <= w.gate_keep
    assert np.all(np.isneginf(thr[:, :, few]))
    assert np.all(np.isfinite(thr[:, :, ~few]))
    if (~few).any():
        Q, K, _, _ = synth.make_inputs(w)
        rng = np.random.default_rng(1)
        blocks = [(0, 0, w.nb - 1), (w.B - 1, w.Hq - 1, w.gate_keep)]
        blocks += [(int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(w.gate_keep, w.nb)))
                   for _ in range(4)]
        ref = oracle.calibrate_thresholds(Q, K, w.blk, w.gate_keep, blocks=blocks)
        for (b, h, j) in blocks:
            assert thr[b, h, j] == ref[b, h, j], (b, h, j)
