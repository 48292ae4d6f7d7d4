"""Failure detection on the GPU without a fault: every wait of the attention
kernels is bounded, and a wait that runs out makes the kernel give up and
report PBS_ERR_TIMEOUT through the device error word while the context stays
usable.  The test hook withholds the "query tile landed" arrival (a flag that
nothing then sets) and shortens the role waits, so the MMA role's first wait
runs out; the next launch with the hook off must give the same results as a
clean run."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import permuted_block_sparse_b200 as pbs
from permuted_block_sparse_b200 import _binding, synth

from gpu_util import LSE_MAX_ABS, assert_close, dev, pack_lists

pytestmark = pytest.mark.gpu

W = synth.Workload("fail", B=1, Hq=4, Hkv=1, N=2048, d=128, blk=128, seg=512, mode="topk", density=0.3,
                   stripe_frac=0.01)


@pytest.fixture(scope="module")
def case():
    Q, K, V, _ = synth.make_inputs(W)
    perm = oracle.permute(Q, K, W.blk, W.seg)
    counts, lists = oracle.select(Q, K, perm, W.blk, W.seg, "topk", density=W.density)
    c_d, idx_d = pack_lists(counts, lists, max(1, int(counts.max())))
    return Q, K, V, perm, lists, c_d, idx_d


@pytest.mark.parametrize("kind", ["one_cta", "cta_pair", "early_stop"])
def test_timed_out_wait_reports_and_next_launch_is_clean(case, kind):
    Q, K, V, perm, lists, c_d, idx_d = case
    Qd, Kd, Vd, pd = dev(Q), dev(K), dev(V), torch.from_numpy(perm).cuda()

    def run():
        if kind == "early_stop":
            return pbs.pbs_attn_fwd_early_stop(Qd, Kd, Vd, pd, c_d, idx_d, W.blk, W.seg, 0.0)
        return pbs.pbs_attn_fwd(Qd, Kd, Vd, pd, c_d, idx_d, W.blk, W.seg, cta_pair=kind == "cta_pair")

    O_clean, L_clean = run()
    pbs.pbs_check_device()
    try:
        _binding.test_inject_timeout(256)
        run()
        with pytest.raises(pbs.PbsError) as e:
            pbs.pbs_check_device()
        assert e.value.code == -5                  # PBS_ERR_TIMEOUT
    finally:
        _binding.test_inject_timeout(0)
    pbs.pbs_check_device()                         # the word was read and cleared
    O, L = run()
    pbs.pbs_check_device()
    assert torch.equal(O, O_clean) and torch.equal(L, L_clean)
    O_ref, L_ref = oracle.attn(Q, K, V, perm, lists, W.blk, W.seg)
    assert_close(O, O_ref, what=kind)
    assert np.max(np.abs(L.cpu().numpy() - L_ref)) <= LSE_MAX_ABS
