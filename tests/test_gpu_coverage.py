"""Attention coverage measured on the GPU -- exp(LSE over a block's key set
minus LSE over all its causal keys), both LSEs from pbs_attn_fwd -- against
the oracle's explicit mass shares ("Sparser Block-Sparse Attention via Token
Permutation", Key Results: permuting keys raises the coverage of a given
number of blocks)."""
import math

import numpy as np
import pytest
import torch

import oracle
import permuted_block_sparse_b200 as pbs
from permuted_block_sparse_b200 import synth

from gpu_util import dev, pack_lists, workload_inputs

pytestmark = pytest.mark.gpu
COVERAGE_ABS = 3e-3      # two LSEs within 1e-3 each: exp(2e-3) - 1 < 2.1e-3


def _gpu_coverage(w, Q, K, V, perm, counts, lists):
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    cap = max(1, int(counts.max()))
    c_d, i_d = pack_lists(counts, lists, cap)
    _, l_sel = pbs.pbs_attn_fwd(Qd, Kd, Vd, torch.from_numpy(perm).cuda(), c_d, i_d, w.blk, w.seg)
    ident = torch.arange(w.N, dtype=torch.int32, device="cuda").expand(w.B, w.Hkv, w.N).contiguous()
    nb = w.nb
    dc = torch.arange(nb, dtype=torch.int32, device="cuda").expand(w.B, w.Hq, nb).contiguous()
    di = torch.arange(max(nb - 1, 1), dtype=torch.int32, device="cuda").expand(w.B, w.Hq, nb, max(nb - 1, 1))
    _, l_all = pbs.pbs_attn_fwd(Qd, Kd, Vd, ident, dc, di.contiguous(), w.blk, w.blk)
    pbs.pbs_check_device()
    return torch.exp(l_sel - l_all).cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("shape", [(1, 4, 2, 2048, 128, 128, 512, 0.25), (1, 2, 1, 1024, 64, 64, 256, 0.3)])
def test_coverage_matches_oracle(shape):
    B, Hq, Hkv, N, d, blk, seg, dens = shape
    w = synth.Workload("cov", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, blk=blk, seg=seg, mode="topk", density=dens,
                       stripe_frac=0.01)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, blk, seg)
    counts, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=dens)
    cov = _gpu_coverage(w, Q, K, V, perm, counts, lists)
    scale = 1.0 / math.sqrt(d)
    for b in range(B):
        for h in range(Hq):
            for i in range(N // blk):
                ref = oracle.coverage_block(Q, K, perm, lists.get((b, h, i), []), b, h, i, blk, seg, scale)
                got = cov[b, h, i * blk:(i + 1) * blk]
                assert np.max(np.abs(got - ref)) <= COVERAGE_ABS, (b, h, i)


def test_permutation_raises_coverage_on_stripe_inputs():
    """On the planted-stripe inputs the permuted selection covers more of the
    attention mass than the same top-k rule on the natural key order."""
    w, Q, K, V = workload_inputs("gqa_8k_band")
    perm = oracle.permute(Q, K, w.blk, w.seg, w.n_sink)
    nat = np.broadcast_to(np.arange(w.N, dtype=np.int32), perm.shape).copy()
    c_p, l_p = oracle.select(Q, K, perm, w.blk, w.seg, "topk", density=w.density, band=w.band)
    c_n, l_n = oracle.select(Q, K, nat, w.blk, w.seg, "topk", density=w.density, band=w.band)
    cov_p = _gpu_coverage(w, Q, K, V, perm, c_p, l_p)
    cov_n = _gpu_coverage(w, Q, K, V, nat, c_n, l_n)
    late = slice(w.seg, None)                  # rows with candidates to choose from
    assert cov_p[:, :, late].mean() > cov_n[:, :, late].mean()
