"""GPU parity of S2O's query permutation ("S2O: Early Stopping for Sparse
Attention via Online Permutation", Technical Summary, 1. Online Permutation
via Index-Driven Loading, Query Permutation): pbs_permute_queries against
oracle.permute_queries (bit-exact), pbs_select_qperm against the oracle's
selection on the gathered queries (bit-exact), and pbs_attn_fwd_qperm
against oracle.attn_qperm (O / LSE within tolerance, written back at the
queries' original positions)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import permuted_block_sparse_b200 as pbs
from permuted_block_sparse_b200 import synth

from gpu_util import (LSE_MAX_ABS, assert_block_scores_exact, assert_close, assert_tau_margins, dev, pack_lists,
                      workload_inputs)

pytestmark = pytest.mark.gpu

SHAPES = [
    synth.Workload("qp_gqa", B=1, Hq=8, Hkv=2, N=4096, d=128, blk=128, seg=1024, mode="topk", density=0.25,
                   stripe_frac=0.01),
    synth.Workload("qp_mha64", B=2, Hq=2, Hkv=2, N=1984, d=64, blk=64, seg=512, mode="topk", density=0.3,
                   stripe_frac=0.02),                       # ragged last segment (448 queries)
    synth.Workload("qp_odd_heads", B=1, Hq=3, Hkv=1, N=2048, d=128, blk=64, seg=256, mode="topk", density=0.3,
                   stripe_frac=0.02, c_lo=3.0, c_hi=6.0),    # an odd head count: one CTA serves a single head
]


def _qperm_gpu(w, Qd, Kd):
    qp = pbs.pbs_permute_queries(Qd, Kd, w.blk, w.seg)
    pbs.pbs_check_device()
    return qp


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_permute_queries_bit_exact(w):
    Q, K, V, _ = synth.make_inputs(w)
    got = _qperm_gpu(w, dev(Q), dev(K)).cpu().numpy()
    assert np.array_equal(got, oracle.permute_queries(Q, K, w.seg))


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
@pytest.mark.parametrize("mode", ["topk", "tau"])
def test_select_qperm_bit_exact(w, mode):
    Q, K, V, _ = synth.make_inputs(w)
    qperm = oracle.permute_queries(Q, K, w.seg)
    perm = oracle.permute(Q, K, w.blk, w.seg)
    Qp = oracle.gather_queries(Q, qperm)
    assert_block_scores_exact(Qp, K, perm, w.blk)
    tau = 0.8
    trace = {}
    counts_ref, lists_ref = oracle.select(Qp, K, perm, w.blk, w.seg, mode, density=w.density, tau=tau, trace=trace)
    if mode == "tau":
        assert_tau_margins(trace, tau)
    c, idx = pbs.pbs_select_qperm(dev(Q), dev(K), torch.from_numpy(perm).cuda(), torch.from_numpy(qperm).cuda(),
                                  w.blk, w.seg, mode, tau if mode == "tau" else w.density)
    pbs.pbs_check_device()
    c, idx = c.cpu().numpy(), idx.cpu().numpy()
    assert np.array_equal(c, counts_ref)
    for key, arr in lists_ref.items():
        assert list(idx[key][:c[key]]) == list(arr), key


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_attn_qperm_full(w):
    """The whole GPU path (query permutation, selection, attention) on the
    oracle's permutations and lists, every row against oracle.attn_qperm."""
    Q, K, V, _ = synth.make_inputs(w)
    qperm = oracle.permute_queries(Q, K, w.seg)
    perm = oracle.permute(Q, K, w.blk, w.seg)
    counts, lists = oracle.select(oracle.gather_queries(Q, qperm), K, perm, w.blk, w.seg, "topk",
                                  density=w.density)
    c_d, idx_d = pack_lists(counts, lists, max(1, int(counts.max())))
    O, L = pbs.pbs_attn_fwd_qperm(dev(Q), dev(K), dev(V), torch.from_numpy(perm).cuda(),
                                  torch.from_numpy(qperm).cuda(), c_d, idx_d, w.blk, w.seg)
    pbs.pbs_check_device()
    O_ref, L_ref = oracle.attn_qperm(Q, K, V, perm, qperm, lists, w.blk, w.seg)
    assert_close(O, O_ref, what=w.name)
    assert np.max(np.abs(L.cpu().numpy() - L_ref)) <= LSE_MAX_ABS


def test_attn_qperm_identity_is_the_natural_kernel():
    """With the identity query permutation the path is the natural-order
    forward, bit for bit."""
    w = SHAPES[0]
    Q, K, V, _ = synth.make_inputs(w)
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    perm = pbs.pbs_permute(Qd, Kd, w.blk, w.seg)
    c, idx = pbs.pbs_select(Qd, Kd, perm, w.blk, w.seg, "topk", w.density)
    ident = torch.arange(w.N, dtype=torch.int32, device="cuda").expand(w.B, w.Hq, w.N).contiguous()
    O1, L1 = pbs.pbs_attn_fwd(Qd, Kd, Vd, perm, c, idx, w.blk, w.seg)
    O2, L2 = pbs.pbs_attn_fwd_qperm(Qd, Kd, Vd, perm, ident, c, idx, w.blk, w.seg)
    pbs.pbs_check_device()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)


def test_qperm_entry_outside_its_segment_is_flagged():
    w = SHAPES[0]
    Q, K, V, _ = synth.make_inputs(w)
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    perm = pbs.pbs_permute(Qd, Kd, w.blk, w.seg)
    qp = pbs.pbs_permute_queries(Qd, Kd, w.blk, w.seg)
    c, idx = pbs.pbs_select_qperm(Qd, Kd, perm, qp, w.blk, w.seg, "topk", w.density)
    pbs.pbs_check_device()
    bad = qp.clone()
    bad[0, 3, 5] = w.N + 7                       # outside every segment
    pbs.pbs_attn_fwd_qperm(Qd, Kd, Vd, perm, bad, c, idx, w.blk, w.seg)
    with pytest.raises(pbs.PbsError) as e:
        pbs.pbs_check_device()
    assert e.value.code == -6
    pbs.pbs_select_qperm(Qd, Kd, perm, bad, w.blk, w.seg, "topk", w.density)
    with pytest.raises(pbs.PbsError) as e:
        pbs.pbs_check_device()
    assert e.value.code == -6


def test_qperm_32k_pipeline_sampled():
    """The 32K shape through the whole GPU path (permute, permute queries,
    select, attention); permutations and lists bit-exact against the oracle
    on the sampled blocks, O and LSE of the sampled blocks within tolerance
    at the queries' original positions."""
    w, Q, K, V = workload_inputs("s2o_32k_qperm")
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    perm = pbs.pbs_permute(Qd, Kd, w.blk, w.seg)
    qp = pbs.pbs_permute_queries(Qd, Kd, w.blk, w.seg)
    c, idx = pbs.pbs_select_qperm(Qd, Kd, perm, qp, w.blk, w.seg, "topk", w.density)
    O, L = pbs.pbs_attn_fwd_qperm(Qd, Kd, Vd, perm, qp, c, idx, w.blk, w.seg)
    pbs.pbs_check_device()
    perm_np, qp_np = perm.cpu().numpy(), qp.cpu().numpy()
    assert np.array_equal(perm_np, oracle.permute(Q, K, w.blk, w.seg))
    assert np.array_equal(qp_np, oracle.permute_queries(Q, K, w.seg))
    blocks = [(0, h, i) for h in (0, 13, 31) for i in (0, 15, 16, 100, 255)]
    Qp = oracle.gather_queries(Q, qp_np)
    counts_ref, lists_ref = oracle.select(Qp, K, perm_np, w.blk, w.seg, "topk", density=w.density, rows=blocks)
    c_np, idx_np = c.cpu().numpy(), idx.cpu().numpy()
    O_np, L_np = O.float().cpu().numpy().astype(np.float64), L.cpu().numpy()
    scale = 1.0 / np.sqrt(w.d)
    for (b, h, i) in blocks:
        assert c_np[b, h, i] == counts_ref[b, h, i]
        listed = idx_np[b, h, i, :c_np[b, h, i]]
        assert list(listed) == list(lists_ref[(b, h, i)])
        o_ref, l_ref = oracle.attn_block_qperm(Q, K, V, perm_np, qp_np, listed, b, h, i, w.blk, w.seg, scale)
        pos = qp_np[b, h, i * w.blk:(i + 1) * w.blk]
        assert_close(torch.from_numpy(O_np[b, h, pos]), o_ref, what=str((b, h, i)))
        assert np.max(np.abs(L_np[b, h, pos] - l_ref)) <= LSE_MAX_ABS
