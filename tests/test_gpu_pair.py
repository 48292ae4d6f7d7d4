"""GPU parity of the CTA-pair attention kernel (PBS_ATTN_CTA_PAIR): four
query heads of a KV head per cluster of two CTAs, MMAs spanning both.

It computes each head's tiles in the same order with the same arithmetic as
the one-CTA kernel, so its O and LSE must be bit-identical to it; it must
match the fp64 oracle within the usual tolerance; and a head must take
nothing from a tile it does not list even though the pair runs that tile's
MMAs for a sibling head (NaN planted in such rows must not reach it)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import permuted_block_sparse_b200 as pbs
from permuted_block_sparse_b200 import synth

from gpu_util import LSE_MAX_ABS, assert_close, dev, pack_lists

pytestmark = pytest.mark.gpu

CASES = [
    synth.Workload("pq_small", B=1, Hq=8, Hkv=2, N=2048, d=128, blk=128, seg=512, mode="topk", density=0.3,
                   stripe_frac=0.01),
    synth.Workload("pq_g8_b2", B=2, Hq=8, Hkv=1, N=4096, d=128, blk=128, seg=1024, mode="topk", density=0.2,
                   stripe_frac=0.01),
    synth.Workload("pq_tau", B=1, Hq=8, Hkv=2, N=4096, d=128, blk=128, seg=1024, mode="tau", tau=0.9,
                   stripe_frac=0.01, c_lo=3.0, c_hi=6.0),
    synth.Workload("pq_ragged", B=1, Hq=4, Hkv=1, N=2944, d=128, blk=128, seg=1024, mode="topk", density=0.25,
                   stripe_frac=0.01, n_sink=128),
]


def _lists_gpu(w, Qd, Kd):
    dt = w.tau if w.mode == "tau" else w.density
    perm = pbs.pbs_permute(Qd, Kd, w.blk, w.seg, w.n_sink)
    c, idx = pbs.pbs_select(Qd, Kd, perm, w.blk, w.seg, w.mode, dt, w.band, w.n_sink)
    pbs.pbs_check_device()
    return perm, c, idx


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_pair_bit_identical_to_one_cta(w):
    Q, K, V, _ = synth.make_inputs(w)
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    perm, c, idx = _lists_gpu(w, Qd, Kd)
    st1 = torch.zeros(2, dtype=torch.int64, device="cuda")
    st2 = torch.zeros(2, dtype=torch.int64, device="cuda")
    O1, L1 = pbs.pbs_attn_fwd(Qd, Kd, Vd, perm, c, idx, w.blk, w.seg, stats=st1)
    O2, L2 = pbs.pbs_attn_fwd(Qd, Kd, Vd, perm, c, idx, w.blk, w.seg, stats=st2, cta_pair=True)
    pbs.pbs_check_device()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
    assert st1.tolist() == st2.tolist()


def test_pair_matches_oracle():
    w = CASES[0]
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, w.blk, w.seg, w.n_sink)
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, "topk", density=w.density)
    c_d, idx_d = pack_lists(counts, lists, max(1, int(counts.max())))
    O, L = pbs.pbs_attn_fwd(dev(Q), dev(K), dev(V), torch.from_numpy(perm).cuda(), c_d, idx_d, w.blk, w.seg,
                            cta_pair=True)
    pbs.pbs_check_device()
    O_ref, L_ref = oracle.attn(Q, K, V, perm, lists, w.blk, w.seg)
    assert_close(O, O_ref, what="pair")
    assert np.max(np.abs(L.cpu().numpy() - L_ref)) <= LSE_MAX_ABS


def test_pair_head_takes_nothing_from_sibling_tiles():
    """NaN in every K/V row outside one head's key set (rows its three
    sibling heads may still list, so the pair runs MMAs over them) must leave
    that head's block bit-identical: the PV leaves the head's output rows
    untouched for tiles it does not list."""
    w = synth.Workload("pq_nan", B=1, Hq=4, Hkv=1, N=4096, d=128, blk=128, seg=512, mode="topk", density=0.15,
                       stripe_frac=0.01)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, w.blk, w.seg)
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, "topk", density=0.15)
    c_d, idx_d = pack_lists(counts, lists, max(1, int(counts.max())))
    pd = torch.from_numpy(perm).cuda()
    O0, _ = pbs.pbs_attn_fwd(dev(Q), dev(K), dev(V), pd, c_d, idx_d, w.blk, w.seg, cta_pair=True)
    checked = 0
    for (h, i) in ((0, w.nb - 1), (1, 20), (3, 17)):
        used = np.zeros(w.N, bool)
        for pb in lists[(0, h, i)]:
            used[perm[0, 0, pb * w.blk:(pb + 1) * w.blk]] = True
        used[(i * w.blk // w.seg) * w.seg:(i + 1) * w.blk] = True
        # the case is only meaningful where a sibling lists a tile this head does not
        sib = set()
        for hh in range(w.Hq):
            if hh != h:
                sib |= set(int(x) for x in lists[(0, hh, i)])
        if not sib - set(int(x) for x in lists[(0, h, i)]):
            continue
        checked += 1
        K2, V2 = K.copy(), V.copy()
        K2[0, 0, ~used] = np.nan
        V2[0, 0, ~used] = np.nan
        O1, _ = pbs.pbs_attn_fwd(dev(Q), dev(K2), dev(V2), pd, c_d, idx_d, w.blk, w.seg, cta_pair=True)
        sl = slice(i * w.blk, (i + 1) * w.blk)
        assert torch.equal(O0[0, h, sl], O1[0, h, sl]), (h, i)
    pbs.pbs_check_device()
    assert checked >= 1
