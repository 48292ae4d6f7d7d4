"""GPU parity of the SampleAttention-style selector ("SampleAttention",
Technical Deep Dive, Stage 1 Trunk Sampling and Stage 2 Score-Based
Filtering) against the fp64 oracle.

The kernel's probabilities are fp32 (summed in fp64), the oracle's fp64, so
a column or slash cut is only compared where the oracle's decision has room:
the accumulated score at the cut lies at least 1e-6 (relative) from the
target on both sides, and the last kept and first dropped scores differ by
at least 2e-6 (relative); the kernel's scores carry relative errors of a few
1e-7.  With a target of 1 there is no cut (every key with a positive score
is kept).  Heads meeting that are compared list for list,
bit-exact; their attention runs through pbs_attn_fwd with the identity
permutation against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import permuted_block_sparse_b200 as pbs
from permuted_block_sparse_b200 import synth

from gpu_util import LSE_MAX_ABS, assert_close, dev, pack_lists, workload_inputs

pytestmark = pytest.mark.gpu
MARGIN_SUM = 1e-6
MARGIN_GAP = 2e-6


def _clear(tr, alpha):
    if alpha >= 1.0:
        return True
    for (before, after, goal, last, nxt) in tr:
        if abs(after - goal) < MARGIN_SUM * goal or abs(goal - before) < MARGIN_SUM * goal:
            return False
        if np.isfinite(nxt) and (last - nxt) < MARGIN_GAP * last:
            return False
    return True


def _compare(w, Q, K, alpha, min_heads):
    trace = {}
    counts, lists = oracle.select_sample(Q, K, w.blk, w.seg, alpha, trace=trace)
    c_d, i_d = pbs.pbs_select(dev(Q), dev(K), None, w.blk, w.seg, "sample", alpha)
    pbs.pbs_check_device()
    c_g, i_g = c_d.cpu().numpy(), i_d.cpu().numpy()
    heads = [bh for bh, tr in trace.items() if _clear(tr, alpha)]
    assert len(heads) >= min_heads, f"only {len(heads)} heads clear of the cut"
    for (b, h) in heads:
        for i in range(w.nb):
            arr = lists[(b, h, i)]
            assert int(c_g[b, h, i]) == arr.size, (b, h, i)
            assert i_g[b, h, i, :arr.size].tolist() == arr.tolist(), (b, h, i)
    return counts, lists, heads


@pytest.mark.parametrize("shape,alpha", [((1, 4, 2, 2048, 128, 128, 512), 0.9),
                                         ((2, 2, 1, 1024, 64, 64, 256), 0.8),
                                         ((1, 2, 1, 1536, 128, 128, 512), 1.0),
                                         ((1, 2, 1, 40960, 64, 128, 4096), 0.7)])
def test_sample_lists_match_oracle(shape, alpha):
    """Small shapes, and one with N > 32768 (the cut re-reads its scores
    from global memory instead of keeping them on chip)."""
    B, Hq, Hkv, N, d, blk, seg = shape
    w = synth.Workload("smp", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, blk=blk, seg=seg, mode="topk",
                       stripe_frac=0.01, c_lo=3.0, c_hi=6.0)
    Q, K, V, _ = synth.make_inputs(w)
    counts, lists, heads = _compare(w, Q, K, alpha, min_heads=max(1, (B * Hq) // 2))
    # attention over the sampled block lists, identity permutation
    ident = np.broadcast_to(np.arange(N, dtype=np.int32), (B, Hkv, N)).copy()
    cap = max(1, int(counts.max()))
    c_d, i_d = pack_lists(counts, lists, cap)
    O, L = pbs.pbs_attn_fwd(dev(Q), dev(K), dev(V), torch.from_numpy(ident).cuda(), c_d, i_d, blk, seg)
    pbs.pbs_check_device()
    O_ref, L_ref = oracle.attn(Q, K, V, ident, lists, blk, seg)
    assert_close(O, O_ref, what=str(shape))
    assert np.nanmax(np.abs(L.cpu().numpy() - L_ref)) <= LSE_MAX_ABS


@pytest.mark.parametrize("alpha", [0.5, 0.95])
def test_sample_lists_8k_workload(alpha):
    w, Q, K, V = workload_inputs("gqa_8k_band")
    _compare(w, Q, K, alpha, min_heads=(w.B * w.Hq) // 2)


def test_sample_32k_workload_sampled():
    """The benchmark's 32K SampleAttention workload in the launch
    configuration the benchmark times: the selector over all heads, then
    attention over its lists.  Two query heads' lists are compared with the
    oracle's (bit-exact where their cuts have room), and six query blocks of
    each head with the oracle's attention over the GPU's own lists."""
    w, Q, K, V = workload_inputs("sample_32k_local")
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    cap = pbs.select_capacity(w.N, w.blk, w.seg, "sample", w.tau)
    c_d, i_d = pbs.pbs_select(Qd, Kd, None, w.blk, w.seg, "sample", w.tau, cap=cap)
    ident = torch.arange(w.N, dtype=torch.int32, device="cuda").expand(w.B, w.Hkv, w.N).contiguous()
    O, L = pbs.pbs_attn_fwd(Qd, Kd, Vd, ident, c_d, i_d, w.blk, w.seg)
    pbs.pbs_check_device()
    c_g, i_g = c_d.cpu().numpy(), i_d.cpu().numpy()
    # the selection is sparse on these inputs
    spb = w.seg // w.blk
    cand = sum(oracle.n_candidates(i, w.blk, w.seg) for i in range(w.nb)) * w.B * w.Hq
    assert 0 < c_g.sum() < 0.5 * cand
    ident_np = np.broadcast_to(np.arange(w.N, dtype=np.int32), (w.B, w.Hkv, w.N)).copy()
    compared = 0
    for h in (0, 21):
        trace = {}
        _, lists = oracle.select_sample(Q, K, w.blk, w.seg, w.tau, rows=[(0, h, i) for i in range(w.nb)],
                                        trace=trace)
        if _clear(trace[(0, h)], w.tau):
            compared += 1
            for i in range(w.nb):
                arr = lists[(0, h, i)]
                assert int(c_g[0, h, i]) == arr.size, (h, i)
                assert i_g[0, h, i, :arr.size].tolist() == arr.tolist(), (h, i)
        blocks = [(0, h, int(i)) for i in np.linspace(spb, w.nb - 1, 6).round()]
        gl = {key: i_g[key][:c_g[key]].copy() for key in blocks}
        ref = oracle.attn_blocks(Q, K, V, ident_np, gl, w.blk, w.seg, blocks)
        for (b, hh, i), (o_ref, l_ref) in ref.items():
            r = slice(i * w.blk, (i + 1) * w.blk)
            assert_close(O[b, hh, r], o_ref, what=f"head {hh} block {i}")
            assert np.nanmax(np.abs(L[b, hh, r].cpu().numpy() - l_ref)) <= LSE_MAX_ABS
    assert compared >= 1
