"""Write the gate thresholds of the gating workloads (offline calibration).

The block-max gating method calibrates its per-(layer, head, position)
thresholds offline so that roughly the top-k key blocks of each query block
are kept ("Block Sparse Flash Attention", Approach).  Here the fp64 oracle
computes, for every (batch, query head, query block) of each gating
workload's seeded synthetic inputs, the 64th-largest exact tile maximum of
raw q.k (-inf when the block has at most 64 causal tiles) and stores them as
float32 (the values are multiples of 2^-6 below 2^18 in magnitude, so fp32
holds them exactly).

Run from the repository root:  python tests/golden/make_gate_thresholds.py
"""
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from permuted_block_sparse_b200 import synth  # noqa: E402


def main(names=("gate_b8_2k", "gate_b8_4k", "gate_b1_64k")):
    for name in names:
        w = synth.WORKLOADS[name]
        t0 = time.time()
        Q, K, V, _ = synth.make_inputs(w)
        thr = oracle.calibrate_thresholds(Q, K, w.blk, w.gate_keep)
        t32 = thr.astype(np.float32)
        assert np.array_equal(t32.astype(np.float64), thr)
        np.save(os.path.join(HERE, f"gate_thr_{name}.npy"), t32)
        print(f"{name}: {thr.shape} thresholds in {time.time() - t0:.0f} s", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:] or ("gate_b8_2k", "gate_b8_4k", "gate_b1_64k"))
