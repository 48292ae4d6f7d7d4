"""GPU parity of the index path: pbs_permute and pbs_select against the fp64
oracle, bit-exact, on seeded lattice inputs whose scores are exactly
representable (asserted before each comparison)."""
import numpy as np
import pytest
import torch

import oracle
import permuted_block_sparse_b200 as pbs
from permuted_block_sparse_b200 import synth

from gpu_util import (assert_block_scores_exact, assert_key_scores_exact, assert_tau_margins, dev,
                      workload_inputs)

pytestmark = pytest.mark.gpu

FULL = ["single_head_1k", "gqa_8k_band", "llama8b_32k_tau", "llama8b_128k_sink"]


@pytest.mark.parametrize("name", FULL)
def test_permute_bit_exact(name):
    w, Q, K, V = workload_inputs(name)
    assert_key_scores_exact(Q, K, w.blk)
    ref = oracle.permute(Q, K, w.blk, w.seg, w.n_sink)
    got = pbs.pbs_permute(dev(Q), dev(K), w.blk, w.seg, w.n_sink)
    pbs.pbs_check_device()
    assert np.array_equal(got.cpu().numpy(), ref)


@pytest.mark.parametrize("shape", [
    # B, Hq, Hkv, N, d, blk, seg, n_sink   (ragged last segment; GQA; d=64)
    (2, 6, 2, 1280, 64, 64, 512, 0),
    (1, 4, 1, 896, 128, 128, 384, 7),
    (1, 2, 2, 256, 128, 64, 64, 300),
])
def test_permute_ragged_and_small(shape):
    B, Hq, Hkv, N, d, blk, seg, n_sink = shape
    Q = synth.random_lattice((B, Hq, N, d), 1, 2.0)
    K = synth.random_lattice((B, Hkv, N, d), 2, 2.0)
    K[..., :5] = np.round(K[..., :5] / 4)      # encourage score ties
    assert_key_scores_exact(Q, K, blk)
    ref = oracle.permute(Q, K, blk, seg, n_sink)
    got = pbs.pbs_permute(dev(Q), dev(K), blk, seg, n_sink)
    pbs.pbs_check_device()
    assert np.array_equal(got.cpu().numpy(), ref)


def test_permute_strided_views():
    """[B, N, H, D] storage viewed as [B, H, N, D] (non-contiguous heads)."""
    B, Hq, Hkv, N, d, blk, seg = 1, 4, 2, 1024, 128, 128, 512
    Q = synth.random_lattice((B, Hq, N, d), 3)
    K = synth.random_lattice((B, Hkv, N, d), 4)
    Qd = dev(np.transpose(Q, (0, 2, 1, 3))).transpose(1, 2)
    Kd = dev(np.transpose(K, (0, 2, 1, 3))).transpose(1, 2)
    assert not Qd.is_contiguous()
    got = pbs.pbs_permute(Qd, Kd, blk, seg)
    assert np.array_equal(got.cpu().numpy(), oracle.permute(Q, K, blk, seg))


def _select_case(w, Q, K, perm, rows=None, **over):
    mode = over.get("mode", w.mode)
    dens = over.get("density", w.density)
    tau = over.get("tau", w.tau)
    band = over.get("band", w.band)
    n_sink = over.get("n_sink", w.n_sink)
    trace = {}
    counts_ref, lists_ref = oracle.select(Q, K, perm, w.blk, w.seg, mode, density=dens, tau=tau,
                                          band=band, n_sink=n_sink, rows=rows, trace=trace)
    if mode == "tau" and tau < 1:
        assert_tau_margins(trace, tau)
    c, idx = pbs.pbs_select(dev(Q), dev(K), torch.from_numpy(perm).cuda(), w.blk, w.seg, mode,
                            tau if mode == "tau" else dens, band, n_sink)
    pbs.pbs_check_device()
    c = c.cpu().numpy()
    idx = idx.cpu().numpy()
    keys = lists_ref.keys() if rows is None else rows
    for key in keys:
        b, h, i = key
        n = c[b, h, i]
        assert n == counts_ref[b, h, i], key
        assert list(idx[b, h, i, :n]) == list(lists_ref[key]), key
    return c


@pytest.mark.parametrize("name", FULL[:3])
def test_select_bit_exact(name):
    w, Q, K, V = workload_inputs(name)
    perm = oracle.permute(Q, K, w.blk, w.seg, w.n_sink)
    assert_block_scores_exact(Q, K, perm, w.blk)
    _select_case(w, Q, K, perm)


def test_select_bit_exact_128k_sampled():
    w, Q, K, V = workload_inputs("llama8b_128k_sink")
    perm = oracle.permute(Q, K, w.blk, w.seg, w.n_sink)
    rng = np.random.default_rng(1)
    rows = [(0, h, int(i)) for h in (0, 9, 22, 31)
            for i in sorted(set(rng.choice(w.nb, 40, replace=False)) | {31, 32, w.nb - 1})]
    G = w.G
    qb = np.abs(oracle.query_block_sums(Q[:, [0, 9, 22, 31]], w.blk))
    kp = np.abs(oracle.permuted_key_block_sums(K, perm, w.blk))
    for t, h in enumerate((0, 9, 22, 31)):
        assert (qb[0, t] @ kp[0, h // G].T).max() < 2.0 ** 18
    _select_case(w, Q, K, perm, rows=rows)


@pytest.mark.parametrize("over", [
    dict(mode="topk", density=1.0),
    dict(mode="topk", density=0.0),
    dict(mode="tau", tau=1.0),
    dict(mode="tau", tau=0.6),
    dict(mode="topk", density=0.25, band=300, n_sink=70),
])
def test_select_edge_cases(over):
    w = synth.Workload("edge", B=2, Hq=4, Hkv=2, N=1536, d=64, blk=64, seg=256, mode="topk",
                       density=0.3, stripe_frac=0.02)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, w.blk, w.seg, over.get("n_sink", 0))
    assert_block_scores_exact(Q, K, perm, w.blk)
    _select_case(w, Q, K, perm, **over)


def test_select_single_segment_has_no_candidates():
    w = synth.Workload("one_seg", B=1, Hq=2, Hkv=1, N=1024, d=128, blk=128, seg=1024, mode="topk",
                       density=0.1)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, w.blk, w.seg)
    c = _select_case(w, Q, K, perm)
    assert c.sum() == 0


def test_select_rejects_perm_outside_segment():
    w = synth.Workload("bad", B=1, Hq=2, Hkv=1, N=1024, d=128, blk=128, seg=256, mode="topk", density=0.5)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, w.blk, w.seg)
    perm[0, 0, 300] = 10                       # crosses into segment 0
    pbs.pbs_select(dev(Q), dev(K), torch.from_numpy(perm).cuda(), w.blk, w.seg, "topk", 0.5)
    with pytest.raises(pbs.PbsError) as e:
        pbs.pbs_check_device()
    assert e.value.code == -6
    pbs.pbs_check_device()                     # error word was cleared
