"""GPU parity of the per-query-segment key permutation ("S2O: Early Stopping
for Sparse Attention via Online Permutation", Technical Summary, 1. Online
Permutation via Index-Driven Loading: historical keys scored against each
segment's representative query) and of selection and attention that read
it: permutations and lists bit-exact, O and LSE within the usual
tolerances, early-stopping decisions exact where every gain is clear of the
threshold."""
import numpy as np
import pytest
import torch

import oracle
import permuted_block_sparse_b200 as pbs
from permuted_block_sparse_b200 import synth

from gpu_util import (EXACT_BOUND, LSE_MAX_ABS, assert_close, dev, pack_lists, sample_blocks,
                      workload_inputs)

pytestmark = pytest.mark.gpu
GAIN_MARGIN = 1e-4

SHAPES = [
    # B, Hq, Hkv, N, d, blk, seg, n_sink
    (1, 4, 2, 4096, 128, 128, 512, 0),
    (2, 2, 1, 2048, 64, 64, 256, 64),
    (1, 3, 1, 1664, 128, 128, 512, 0),     # ragged: last segment 128 keys
]


def _inputs(shape, seed=0):
    B, Hq, Hkv, N, d, blk, seg, n_sink = shape
    w = synth.Workload("seg", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, blk=blk, seg=seg, mode="topk", density=0.3,
                       n_sink=n_sink, stripe_frac=0.01, c_lo=3.0, c_hi=6.0, seed=seed)
    Q, K, V, _ = synth.make_inputs(w)
    return w, Q, K, V


def _assert_block_scores_exact(Q, K, perm4, blk):
    qb = np.abs(oracle.query_block_sums(Q, blk))
    G = Q.shape[1] // K.shape[1]
    for s in range(perm4.shape[2]):
        kp = np.abs(oracle.permuted_key_block_sums(K, perm4[:, :, s], blk))
        for b in range(Q.shape[0]):
            for h in range(Q.shape[1]):
                assert (qb[b, h] @ kp[b, h // G].T).max() < EXACT_BOUND


@pytest.mark.parametrize("shape", SHAPES)
def test_permute_segmented_bit_exact(shape):
    w, Q, K, V = _inputs(shape)
    perm = pbs.pbs_permute_segmented(dev(Q), dev(K), w.blk, w.seg, w.n_sink)
    pbs.pbs_check_device()
    ref = oracle.permute_segmented(Q, K, w.blk, w.seg, w.n_sink)
    assert np.array_equal(perm.cpu().numpy(), ref)


def test_permute_segmented_32k_bit_exact():
    w, Q, K, V = workload_inputs("llama8b_32k_tau")
    perm = pbs.pbs_permute_segmented(dev(Q), dev(K), w.blk, w.seg, w.n_sink)
    pbs.pbs_check_device()
    ref = oracle.permute_segmented(Q, K, w.blk, w.seg, w.n_sink)
    assert np.array_equal(perm.cpu().numpy(), ref)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mode,dt,band,order", [("topk", 0.3, 0, False), ("tau", 0.9, 0, False),
                                                ("topk", 0.25, 100, True)])
def test_select_segmented_bit_exact(shape, mode, dt, band, order):
    w, Q, K, V = _inputs(shape)
    perm = oracle.permute_segmented(Q, K, w.blk, w.seg, w.n_sink)
    _assert_block_scores_exact(Q, K, perm, w.blk)
    trace = {} if mode == "tau" else None
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, mode, density=dt, tau=dt, band=band,
                                  n_sink=w.n_sink, trace=trace, list_order="score" if order else "ascending")
    if trace:
        worst = min(min(abs(a - dt), abs(bf - dt)) for bf, a in trace.values())
        assert worst >= 1e-9
    c_d, i_d = pbs.pbs_select(dev(Q), dev(K), torch.from_numpy(perm).cuda(), w.blk, w.seg, mode, dt, band,
                              w.n_sink, score_order=order)
    pbs.pbs_check_device()
    c_g, i_g = c_d.cpu().numpy(), i_d.cpu().numpy()
    assert np.array_equal(c_g, counts)
    for (b, h, i), arr in lists.items():
        assert i_g[b, h, i, :arr.size].tolist() == arr.tolist(), (b, h, i)


@pytest.mark.parametrize("shape", SHAPES)
def test_attn_segmented_matches_oracle(shape):
    w, Q, K, V = _inputs(shape)
    perm = oracle.permute_segmented(Q, K, w.blk, w.seg, w.n_sink)
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, "topk", density=0.3, n_sink=w.n_sink)
    O_ref, L_ref = oracle.attn(Q, K, V, perm, lists, w.blk, w.seg)
    cap = max(1, int(counts.max()))
    c_d, i_d = pack_lists(counts, lists, cap)
    O, L = pbs.pbs_attn_fwd(dev(Q), dev(K), dev(V), torch.from_numpy(perm).cuda(), c_d, i_d, w.blk, w.seg)
    pbs.pbs_check_device()
    assert_close(O, O_ref, what=str(shape))
    assert np.nanmax(np.abs(L.cpu().numpy() - L_ref)) <= LSE_MAX_ABS


def test_s2o_pipeline_segmented_early_stop():
    """Segmented permutation, visiting-order selection of every candidate and
    early stopping, all on the GPU, against the oracle on the same steps."""
    w, Q, K, V = _inputs((1, 4, 2, 4096, 128, 128, 512, 0), seed=3)
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    perm_d = pbs.pbs_permute_segmented(Qd, Kd, w.blk, w.seg)
    c_d, i_d = pbs.pbs_select(Qd, Kd, perm_d, w.blk, w.seg, "topk", 1.0, score_order=True)
    perm = perm_d.cpu().numpy()
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, "topk", density=1.0, list_order="score")
    blocks = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.nb)]
    full = {}
    oracle.attn_early_stop(Q, K, V, perm, lists, w.blk, w.seg, 0.0, blocks, traces=full)
    gains = np.concatenate([np.asarray(t) for t in full.values() if len(t)])
    tau = None
    for qn in (0.3, 0.4, 0.5, 0.35, 0.45):
        cand = float(np.quantile(gains, qn)) * 1.00037
        tr = {}
        ref = oracle.attn_early_stop(Q, K, V, perm, lists, w.blk, w.seg, cand, blocks, traces=tr)
        if all(abs(g - cand) >= GAIN_MARGIN * cand for t in tr.values() for g in t):
            tau = cand
            break
    assert tau is not None
    st = torch.zeros(2, dtype=torch.int64, device="cuda")
    O, L = pbs.pbs_attn_fwd_early_stop(Qd, Kd, Vd, perm_d, c_d, i_d, w.blk, w.seg, tau, stats=st)
    pbs.pbs_check_device()
    assert np.array_equal(c_d.cpu().numpy(), counts)
    O_ref = np.full((w.B, w.Hq, w.N, w.d), np.nan)
    run = skipped = 0
    for (b, h, i), (o, l, n) in ref.items():
        O_ref[b, h, i * w.blk:(i + 1) * w.blk] = o
        run += len(oracle.diagonal_blocks(i, w.blk, w.seg)) + n
        skipped += len(lists[(b, h, i)]) - n
    assert skipped > 0
    assert (int(st[0]), int(st[1])) == (run, skipped)
    assert_close(O, O_ref, what="s2o segmented")


def test_s2o_segmented_workload_sampled():
    """The 32K segmented S2O workload in the bench's launch configuration;
    sampled blocks against the oracle (blocks with a gain inside the margin
    are left out)."""
    w, Q, K, V = workload_inputs("s2o_32k_segperm")
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    perm_d = pbs.pbs_permute_segmented(Qd, Kd, w.blk, w.seg, w.n_sink)
    c_d, i_d = pbs.pbs_select(Qd, Kd, perm_d, w.blk, w.seg, "topk", w.density, w.band, w.n_sink,
                              score_order=True)
    st = torch.zeros(2, dtype=torch.int64, device="cuda")
    O, L = pbs.pbs_attn_fwd_early_stop(Qd, Kd, Vd, perm_d, c_d, i_d, w.blk, w.seg, w.stop_tau, stats=st)
    pbs.pbs_check_device()
    perm = perm_d.cpu().numpy()
    blocks = sample_blocks(w, [0, 13, 31])
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, "topk", density=1.0, rows=blocks, list_order="score")
    tr = {}
    ref = oracle.attn_early_stop(Q, K, V, perm, lists, w.blk, w.seg, w.stop_tau, blocks, traces=tr)
    O_np = O.float().cpu().numpy().astype(np.float64)
    L_np = L.cpu().numpy()
    compared = 0
    for key, (o, l, n) in ref.items():
        if not all(abs(g - w.stop_tau) >= GAIN_MARGIN * w.stop_tau for g in tr[key]):
            continue
        b, h, i = key
        sl = slice(i * w.blk, (i + 1) * w.blk)
        assert_close(torch.from_numpy(O_np[b, h, sl]), o, what=str(key))
        assert np.max(np.abs(L_np[b, h, sl] - l)) <= LSE_MAX_ABS
        compared += 1
    assert compared >= 15
