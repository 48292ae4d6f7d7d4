"""GPU parity of S2O's visiting order and early stopping against the fp64
oracle ("S2O: Early Stopping for Sparse Attention via Online Permutation",
Technical Summary, 2. Early-Stopping Rule and 3. Kernel Implementation).

Lists in visiting order are compared bit for bit.  The stop decisions are
compared exactly (tiles run and skipped) on inputs where every evaluated
gain is at least 1e-4 relative away from the threshold -- the kernel takes
them in fp32 on its running sums, the oracle in fp64; O and LSE are compared
with the usual tolerances."""
import numpy as np
import pytest
import torch

import oracle
import permuted_block_sparse_b200 as pbs
from permuted_block_sparse_b200 import synth

from gpu_util import (LSE_MAX_ABS, assert_block_scores_exact, assert_close, dev, pack_lists,
                      sample_blocks, workload_inputs)

pytestmark = pytest.mark.gpu
GAIN_MARGIN = 1e-4


def _margins_ok(traces: dict, tau: float) -> bool:
    return all(abs(g - tau) >= GAIN_MARGIN * tau for tr in traces.values() for g in tr)


@pytest.mark.parametrize("name,mode,dt", [("gqa_8k_band", "topk", 0.2), ("single_head_1k", "topk", 0.3),
                                          ("llama8b_32k_tau", "tau", 0.95)])
def test_score_order_lists_bit_exact(name, mode, dt):
    w, Q, K, V = workload_inputs(name)
    perm = oracle.permute(Q, K, w.blk, w.seg, w.n_sink)
    assert_block_scores_exact(Q, K, perm, w.blk)
    rows = None if w.N <= 8192 else sample_blocks(w, [0, 17, 31])
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, mode, density=dt, tau=dt, band=w.band,
                                  n_sink=w.n_sink, rows=rows, list_order="score")
    c_d, i_d = pbs.pbs_select(dev(Q), dev(K), torch.from_numpy(perm).cuda(), w.blk, w.seg, mode, dt, w.band,
                              w.n_sink, score_order=True)
    pbs.pbs_check_device()
    c_g, i_g = c_d.cpu().numpy(), i_d.cpu().numpy()
    keys = rows if rows is not None else list(lists.keys())
    for (b, h, i) in keys:
        n = int(counts[b, h, i])
        assert int(c_g[b, h, i]) == n, (b, h, i)
        assert i_g[b, h, i, :n].tolist() == lists[(b, h, i)].tolist(), (b, h, i)


def _run_es(w, Q, K, V, perm, counts, lists, tau):
    cap = max(1, int(counts.max()))
    c_d, idx_d = pack_lists(counts, lists, cap)
    st = torch.zeros(2, dtype=torch.int64, device="cuda")
    O, L = pbs.pbs_attn_fwd_early_stop(dev(Q), dev(K), dev(V), torch.from_numpy(perm).cuda(), c_d, idx_d,
                                       w.blk, w.seg, tau, stats=st)
    pbs.pbs_check_device()
    return O, L, st


def _pick_tau(Q, K, V, perm, lists, blk, seg, blocks):
    """A threshold inside the range of the gains seen without stopping (so the
    rule fires for some blocks and not for others) whose every evaluated gain
    is clear of it by the margin."""
    full = {}
    oracle.attn_early_stop(Q, K, V, perm, lists, blk, seg, 0.0, blocks, traces=full)
    gains = np.concatenate([np.asarray(t) for t in full.values() if len(t)])
    for q in (0.3, 0.4, 0.5, 0.35, 0.45, 0.25, 0.55):
        tau = float(np.quantile(gains, q)) * 1.00037
        traces = {}
        oracle.attn_early_stop(Q, K, V, perm, lists, blk, seg, tau, blocks, traces=traces)
        if _margins_ok(traces, tau):
            return tau
    raise AssertionError("no threshold with clear margins")


@pytest.mark.parametrize("shape", [
    # B, Hq, Hkv, N, d, blk, seg
    (1, 4, 2, 4096, 128, 128, 512),
    (2, 2, 1, 2048, 64, 64, 256),
    (1, 3, 1, 1536, 128, 64, 384),      # ragged: last segment holds 2 of 6 blocks
])
def test_early_stop_matches_oracle(shape):
    B, Hq, Hkv, N, d, blk, seg = shape
    w = synth.Workload("es", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, blk=blk, seg=seg, mode="topk", density=1.0,
                       stripe_frac=0.01, c_lo=3.0, c_hi=6.0)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, blk, seg)
    counts, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=1.0, list_order="score")
    blocks = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(N // blk)]
    chosen = _pick_tau(Q, K, V, perm, lists, blk, seg, blocks)
    traces = {}
    ref = oracle.attn_early_stop(Q, K, V, perm, lists, blk, seg, chosen, blocks, traces=traces)
    O, L, st = _run_es(w, Q, K, V, perm, counts, lists, chosen)
    O_ref = np.full((B, Hq, N, d), np.nan)
    L_ref = np.full((B, Hq, N), np.nan)
    run = skipped = 0
    for (b, h, i), (o, l, n) in ref.items():
        O_ref[b, h, i * blk:(i + 1) * blk] = o
        L_ref[b, h, i * blk:(i + 1) * blk] = l
        run += len(oracle.diagonal_blocks(i, blk, seg)) + n
        skipped += len(lists[(b, h, i)]) - n
    assert skipped > 0, "the rule never fired"
    assert (int(st[0]), int(st[1])) == (run, skipped)
    assert_close(O, O_ref, what=str(shape))
    assert np.nanmax(np.abs(L.cpu().numpy() - L_ref)) <= LSE_MAX_ABS


def test_early_stop_limits():
    """stop_tau = 0 runs every listed block (equals pbs_attn_fwd's result within
    tolerance and the oracle's sparse attention); a threshold above 1 runs
    exactly one listed block per query block."""
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 2048, 128, 128, 256
    w = synth.Workload("esl", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, blk=blk, seg=seg, mode="topk", density=0.5,
                       stripe_frac=0.01)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, blk, seg)
    counts, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=0.5, list_order="score")
    O, L, st = _run_es(w, Q, K, V, perm, counts, lists, 0.0)
    O_ref, L_ref = oracle.attn(Q, K, V, perm, lists, blk, seg)
    assert_close(O, O_ref, what="tau 0")
    assert int(st[1]) == 0
    O, L, st = _run_es(w, Q, K, V, perm, counts, lists, 1.5)
    first = {k: v[:1] for k, v in lists.items()}
    O_ref, L_ref = oracle.attn(Q, K, V, perm, first, blk, seg)
    assert_close(O, O_ref, what="tau 1.5")
    assert int(st[1]) == int(counts.sum()) - int((counts > 0).sum())


def test_early_stop_repeated_entry_is_flagged():
    B, Hq, Hkv, N, d, blk, seg = 1, 1, 1, 1024, 64, 64, 256
    w = synth.Workload("esr", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, blk=blk, seg=seg, mode="topk", density=1.0)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, blk, seg)
    counts, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=1.0, list_order="score")
    key = (0, 0, N // blk - 1)
    lst = lists[key].copy()
    lst[1] = lst[0]
    lists[key] = lst
    cap = int(counts.max())
    c_d, idx_d = pack_lists(counts, lists, cap)
    pbs.pbs_attn_fwd_early_stop(dev(Q), dev(K), dev(V), torch.from_numpy(perm).cuda(), c_d, idx_d, blk, seg, 0.0)
    with pytest.raises(pbs.PbsError):
        pbs.pbs_check_device()


def test_s2o_workload_sampled():
    """The 32K early-stopping workload in the bench's launch configuration:
    GPU permutation, GPU visiting-order selection of every candidate, early
    stopping at the workload's threshold; sampled blocks against the oracle
    (blocks whose gains come within the margin are skipped)."""
    w, Q, K, V = workload_inputs("s2o_32k_stop")
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    perm_d = pbs.pbs_permute(Qd, Kd, w.blk, w.seg, w.n_sink)
    c_d, i_d = pbs.pbs_select(Qd, Kd, perm_d, w.blk, w.seg, "topk", w.density, w.band, w.n_sink,
                              score_order=True)
    st = torch.zeros(2, dtype=torch.int64, device="cuda")
    O, L = pbs.pbs_attn_fwd_early_stop(Qd, Kd, Vd, perm_d, c_d, i_d, w.blk, w.seg, w.stop_tau, stats=st)
    pbs.pbs_check_device()
    perm = perm_d.cpu().numpy()
    assert np.array_equal(perm, oracle.permute(Q, K, w.blk, w.seg, w.n_sink))
    blocks = sample_blocks(w, [0, 11, 30])
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, "topk", density=1.0, rows=blocks, list_order="score")
    traces = {}
    ref = oracle.attn_early_stop(Q, K, V, perm, lists, w.blk, w.seg, w.stop_tau, blocks, traces=traces)
    O_np = O.float().cpu().numpy().astype(np.float64)
    L_np = L.cpu().numpy()
    compared = 0
    for key, (o, l, n) in ref.items():
        if not _margins_ok({key: traces[key]}, w.stop_tau):
            continue
        b, h, i = key
        sl = slice(i * w.blk, (i + 1) * w.blk)
        assert_close(torch.from_numpy(O_np[b, h, sl]), o, what=str(key))
        assert np.max(np.abs(L_np[b, h, sl] - l)) <= LSE_MAX_ABS
        compared += 1
    assert compared >= 15
    assert int(st[1]) > 0
