"""GPU parity of pbs_attn_fwd against the fp64 oracle, given identical
permutations and block lists: max-abs <= 2e-2 and relative L2 <= 5e-3 on O,
1e-3 on the log-sum-exp; plus properties that hold at any size (unselected
and gated tiles are never read, future keys never matter)."""
import math

import numpy as np
import pytest
import torch

import oracle
import permuted_block_sparse_b200 as pbs
from permuted_block_sparse_b200 import synth

from gpu_util import LSE_MAX_ABS, assert_close, dev, pack_lists, sample_blocks, workload_inputs

pytestmark = pytest.mark.gpu


def _run(w, Q, K, V, perm, counts, lists, gate=None, stats=False):
    cap = max(1, int(counts.max()) if counts.size else 1)
    c_d, idx_d = pack_lists(counts, lists, cap)
    st = torch.zeros(2, dtype=torch.int64, device="cuda") if stats else None
    thr = None if gate is None else torch.from_numpy(gate.astype(np.float32)).cuda()
    O, L = pbs.pbs_attn_fwd(dev(Q), dev(K), dev(V), torch.from_numpy(perm).cuda(), c_d, idx_d,
                            w.blk, w.seg, gate_thr=thr, stats=st)
    pbs.pbs_check_device()
    return O, L, st


def _check_all(w, Q, K, V, perm, counts, lists, gate=None, what=""):
    O_ref, L_ref = oracle.attn(Q, K, V, perm, lists, w.blk, w.seg, gate_thr=gate)
    O, L, _ = _run(w, Q, K, V, perm, counts, lists, gate)
    assert_close(O, O_ref, what=what)
    assert np.nanmax(np.abs(L.cpu().numpy() - L_ref)) <= LSE_MAX_ABS


SHAPES = [
    # B, Hq, Hkv, N, d, blk, seg, density
    (1, 1, 1, 1024, 64, 64, 256, 0.3),
    (2, 4, 2, 1280, 128, 128, 256, 0.4),     # ragged: 10 blocks, last segment of 2
    (1, 2, 1, 768, 128, 64, 192, 0.5),
    (1, 3, 1, 640, 64, 128, 256, 0.35),
    (2, 8, 2, 2048, 128, 128, 512, 0.2),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_attn_small_shapes(shape):
    B, Hq, Hkv, N, d, blk, seg, dens = shape
    w = synth.Workload("s", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, blk=blk, seg=seg, mode="topk", density=dens,
                       stripe_frac=0.02)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, blk, seg)
    counts, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=dens)
    _check_all(w, Q, K, V, perm, counts, lists, what=str(shape))


def test_attn_dense_equals_causal():
    B, Hq, Hkv, N, d, blk, seg = 1, 4, 2, 2048, 128, 128, 128
    w = synth.Workload("dense", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, blk=blk, seg=seg, mode="topk")
    Q, K, V, _ = synth.make_inputs(w)
    perm = np.broadcast_to(np.arange(N, dtype=np.int32), (B, Hkv, N)).copy()
    counts, lists = oracle.dense_lists(B, Hq, N // blk, blk, seg)
    O, _, _ = _run(w, Q, K, V, perm, counts, lists)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q).double(), torch.from_numpy(np.repeat(K, 2, 1)).double(),
        torch.from_numpy(np.repeat(V, 2, 1)).double(), is_causal=True).numpy()
    assert_close(O, ref, what="dense")


@pytest.mark.parametrize("name", ["single_head_1k", "gqa_8k_band"])
def test_attn_workloads_full(name):
    w, Q, K, V = workload_inputs(name)
    perm = oracle.permute(Q, K, w.blk, w.seg, w.n_sink)
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, w.mode, density=w.density, tau=w.tau,
                                  band=w.band, n_sink=w.n_sink)
    _check_all(w, Q, K, V, perm, counts, lists, what=name)


@pytest.mark.parametrize("name,heads", [("llama8b_32k_tau", (0, 13, 31)), ("llama8b_128k_sink", (0, 21))])
def test_attn_workloads_sampled(name, heads):
    """Full-size launch (the configuration the benchmark times); the oracle
    checks every row of a sample of query blocks."""
    w, Q, K, V = workload_inputs(name)
    perm = oracle.permute(Q, K, w.blk, w.seg, w.n_sink)
    blocks = sample_blocks(w, heads)
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, w.mode, density=w.density, tau=w.tau,
                                  band=w.band, n_sink=w.n_sink, rows=blocks)
    # every other row gets the device's own selection so the launch is full size
    c_dev, idx_dev = pbs.pbs_select(dev(Q), dev(K), torch.from_numpy(perm).cuda(), w.blk, w.seg, w.mode,
                                    w.tau if w.mode == "tau" else w.density, w.band, w.n_sink)
    c_np, idx_np = c_dev.cpu().numpy(), idx_dev.cpu().numpy()
    for key in blocks:
        assert c_np[key] == counts[key] and list(idx_np[key][:counts[key]]) == list(lists[key])
    O, L = pbs.pbs_attn_fwd(dev(Q), dev(K), dev(V), torch.from_numpy(perm).cuda(), c_dev, idx_dev,
                            w.blk, w.seg)
    pbs.pbs_check_device()
    ref = oracle.attn_blocks(Q, K, V, perm, lists, w.blk, w.seg, blocks)
    O_np = O.float().cpu().numpy().astype(np.float64)
    L_np = L.cpu().numpy()
    for (b, h, i), (o_ref, l_ref) in ref.items():
        sl = slice(i * w.blk, (i + 1) * w.blk)
        assert_close(torch.from_numpy(O_np[b, h, sl]), o_ref, what=f"{name} {(b, h, i)}")
        assert np.max(np.abs(L_np[b, h, sl] - l_ref)) <= LSE_MAX_ABS


def test_gated_attention_small():
    w = synth.Workload("g", B=2, Hq=4, Hkv=1, N=2048, d=128, blk=128, seg=128, mode="gate", gate_keep=5,
                       stripe_frac=0.01, c_lo=3.0, c_hi=6.0)
    Q, K, V, _ = synth.make_inputs(w)
    perm = np.broadcast_to(np.arange(w.N, dtype=np.int32), (w.B, w.Hkv, w.N)).copy()
    counts, lists = oracle.dense_lists(w.B, w.Hq, w.nb, w.blk, w.seg)
    thr = oracle.calibrate_thresholds(Q, K, w.blk, w.gate_keep)
    O_ref, L_ref = oracle.attn(Q, K, V, perm, lists, w.blk, w.seg, gate_thr=thr)
    O, L, st = _run(w, Q, K, V, perm, counts, lists, gate=thr, stats=True)
    assert_close(O, O_ref, what="gated")
    # executed QK tiles = every causal tile; gated = those below threshold
    n_causal = w.B * w.Hq * w.nb * (w.nb + 1) // 2
    kept = 0
    for b in range(w.B):
        for h in range(w.Hq):
            for i in range(w.nb):
                M = oracle.tile_maxima(Q, K, b, h, i, w.blk)
                kept += 1 + int(np.sum(M[:i] >= thr[b, h, i]))
    assert int(st[0]) == n_causal
    assert int(st[1]) == n_causal - kept


@pytest.mark.parametrize("name", ["gate_b8_2k", "gate_b8_4k"])
def test_gated_attention_short_n_workloads(name):
    """The short-N gating workloads as the bench runs them (B = 8, every
    earlier block listed, the stored offline thresholds).  With at most 32
    causal tiles per row every threshold is -inf, so no tile may be gated:
    the gated run must execute every causal tile, gate none, and give the
    same bits as the run without thresholds; sampled query blocks match the
    oracle (first, last, interior blocks of several heads and batches)."""
    import os
    w, Q, K, V = workload_inputs(name)
    thr = np.load(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", f"gate_thr_{name}.npy"))
    assert np.all(np.isneginf(thr))
    perm = np.broadcast_to(np.arange(w.N, dtype=np.int32), (w.B, w.Hkv, w.N)).copy()
    counts, lists = oracle.dense_lists(w.B, w.Hq, w.nb, w.blk, w.seg)
    O, L, st = _run(w, Q, K, V, perm, counts, lists, gate=thr.astype(np.float64), stats=True)
    n_causal = w.B * w.Hq * w.nb * (w.nb + 1) // 2
    assert int(st[0]) == n_causal and int(st[1]) == 0
    O_plain, L_plain, _ = _run(w, Q, K, V, perm, counts, lists)
    assert torch.equal(O, O_plain) and torch.equal(L, L_plain)
    last = w.nb - 1
    blocks = [(b, h, i) for b in (0, 5, 7) for h in (0, 17, 31) for i in (0, 3, last // 2, last)]
    ref = oracle.attn_blocks(Q, K, V, perm, lists, w.blk, w.seg, blocks, gate_thr=thr.astype(np.float64))
    O_np = O.float().cpu().numpy().astype(np.float64)
    L_np = L.cpu().numpy()
    for (b, h, i), (o_ref, l_ref) in ref.items():
        sl = slice(i * w.blk, (i + 1) * w.blk)
        assert_close(torch.from_numpy(O_np[b, h, sl]), o_ref, what=str((b, h, i)))
        assert np.max(np.abs(L_np[b, h, sl] - l_ref)) <= LSE_MAX_ABS


def test_gated_attention_sampled_calibrated():
    """gate_b8_2k's inputs with thresholds calibrated to keep 5 tiles (so the
    gate does fire at this length): sampled blocks against the oracle."""
    w, Q, K, V = workload_inputs("gate_b8_2k")
    perm = np.broadcast_to(np.arange(w.N, dtype=np.int32), (w.B, w.Hkv, w.N)).copy()
    counts, lists = oracle.dense_lists(w.B, w.Hq, w.nb, w.blk, w.seg)
    blocks = [(b, h, i) for b in (0, 7) for h in (0, 17, 31) for i in (0, 3, 8, 15)]
    thr = oracle.calibrate_thresholds(Q, K, w.blk, 5, blocks=blocks)
    O, L, st = _run(w, Q, K, V, perm, counts, lists, gate=thr, stats=True)
    assert int(st[1]) > 0
    ref = oracle.attn_blocks(Q, K, V, perm, lists, w.blk, w.seg, blocks, gate_thr=thr)
    O_np = O.float().cpu().numpy().astype(np.float64)
    for (b, h, i), (o_ref, _) in ref.items():
        sl = slice(i * w.blk, (i + 1) * w.blk)
        assert_close(torch.from_numpy(O_np[b, h, sl]), o_ref, what=str((b, h, i)))


def test_gated_attention_64k_stored_thresholds():
    """The 64K gating workload as the bench runs it: every earlier block
    listed, the offline thresholds stored beside the tests, identity order.
    Sampled query blocks (all with more than 64 causal tiles but block 0)
    against the oracle; the kernel must gate most tiles."""
    import os
    w, Q, K, V = workload_inputs("gate_b1_64k")
    thr = np.load(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "gate_thr_gate_b1_64k.npy"))
    perm = np.broadcast_to(np.arange(w.N, dtype=np.int32), (w.B, w.Hkv, w.N)).copy()
    counts, lists = oracle.dense_lists(w.B, w.Hq, w.nb, w.blk, w.seg)
    O, L, st = _run(w, Q, K, V, perm, counts, lists, gate=thr.astype(np.float64), stats=True)
    n_causal = w.B * w.Hq * w.nb * (w.nb + 1) // 2
    assert int(st[0]) == n_causal
    # at most keep + ties + the own tile are kept per block with a finite threshold
    assert int(st[1]) > n_causal // 2
    blocks = [(0, 0, 0), (0, 0, 64), (0, 5, 65), (0, 17, 300), (0, 31, w.nb - 1), (0, 12, 449)]
    ref = oracle.attn_blocks(Q, K, V, perm, lists, w.blk, w.seg, blocks, gate_thr=thr.astype(np.float64))
    O_np = O.float().cpu().numpy().astype(np.float64)
    L_np = L.cpu().numpy()
    for (b, h, i), (o_ref, l_ref) in ref.items():
        sl = slice(i * w.blk, (i + 1) * w.blk)
        assert_close(torch.from_numpy(O_np[b, h, sl]), o_ref, what=str((b, h, i)))
        assert np.max(np.abs(L_np[b, h, sl] - l_ref)) <= LSE_MAX_ABS


def test_unvisited_tiles_are_never_read():
    """NaN in every K/V row outside one query block's key set must not reach
    that block's output (bit-identical to the clean run): rows of unlisted
    blocks are never loaded for it.  Other blocks may read those rows, so
    only the target block is compared."""
    w = synth.Workload("nan", B=1, Hq=2, Hkv=1, N=4096, d=128, blk=128, seg=512, mode="topk", density=0.15,
                       stripe_frac=0.01)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, w.blk, w.seg)
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, "topk", density=0.15)
    O0, _, _ = _run(w, Q, K, V, perm, counts, lists)
    for (h, i) in ((0, w.nb - 1), (1, 20)):
        used = np.zeros(w.N, bool)
        for pb in lists[(0, h, i)]:
            used[perm[0, 0, pb * w.blk:(pb + 1) * w.blk]] = True
        used[(i * w.blk // w.seg) * w.seg:(i + 1) * w.blk] = True
        assert (~used).sum() > w.N // 2
        K2, V2 = K.copy(), V.copy()
        K2[0, 0, ~used] = np.nan
        V2[0, 0, ~used] = np.nan
        O1, _, _ = _run(w, Q, K2, V2, perm, counts, lists)
        sl = slice(i * w.blk, (i + 1) * w.blk)
        assert torch.equal(O0[0, h, sl], O1[0, h, sl]), (h, i)


def test_gated_tiles_contribute_nothing():
    """A block whose threshold gates every tile but its own must equal
    attention over its diagonal tile alone, and NaN in the V rows of its gated
    tiles must not reach it (the gated tiles contribute no PV product)."""
    w = synth.Workload("gnan", B=1, Hq=1, Hkv=1, N=1536, d=128, blk=128, seg=128, mode="gate",
                       stripe_frac=0.01)
    Q, K, V, _ = synth.make_inputs(w)
    perm = np.arange(w.N, dtype=np.int32)[None, None].copy()
    counts, lists = oracle.dense_lists(1, 1, w.nb, w.blk, w.seg)
    target = w.nb - 1
    thr = np.full((1, 1, w.nb), -np.inf)
    thr[0, 0, target] = 1e30                   # every tile below it
    O0, _, st = _run(w, Q, K, V, perm, counts, lists, gate=thr, stats=True)
    assert int(st[1]) == target                # all earlier tiles of the target gated
    V2 = V.copy()
    V2[0, 0, :target * w.blk] = np.nan
    O1, _, _ = _run(w, Q, K, V2, perm, counts, lists, gate=thr)
    sl = slice(target * w.blk, (target + 1) * w.blk)
    assert torch.equal(O0[0, 0, sl], O1[0, 0, sl])
    ref = oracle.attn_blocks(Q, K, V, perm, lists, w.blk, w.seg, [(0, 0, target)], gate_thr=thr)
    assert_close(O0[0, 0, sl], ref[(0, 0, target)][0], what="only the diagonal tile")


def test_future_keys_do_not_matter():
    w = synth.Workload("fut", B=1, Hq=2, Hkv=1, N=2048, d=64, blk=64, seg=256, mode="topk", density=0.3,
                       stripe_frac=0.02)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, w.blk, w.seg)
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, "topk", density=0.3)
    O0, _, _ = _run(w, Q, K, V, perm, counts, lists)
    for cut in (700, 1333):
        K2, V2 = K.copy(), V.copy()
        K2[:, :, cut:] = 31.875
        V2[:, :, cut:] = -31.875
        O1, _, _ = _run(w, Q, K2, V2, perm, counts, lists)
        assert torch.equal(O0[:, :, :cut], O1[:, :, :cut])


def test_list_order_does_not_matter():
    w = synth.Workload("ord", B=1, Hq=2, Hkv=1, N=2048, d=128, blk=128, seg=256, mode="topk", density=0.4,
                       stripe_frac=0.02)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, w.blk, w.seg)
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, "topk", density=0.4)
    rng = np.random.default_rng(0)
    shuffled = {k: rng.permutation(v).astype(np.int32) for k, v in lists.items()}
    O0, _, _ = _run(w, Q, K, V, perm, counts, lists)
    O1, _, _ = _run(w, Q, K, V, perm, counts, shuffled)
    O_ref, _ = oracle.attn(Q, K, V, perm, lists, w.blk, w.seg)
    assert_close(O1, O_ref, what="shuffled lists")
    assert (O0.float() - O1.float()).abs().max().item() <= 2e-2


def test_bad_indices_set_device_error_without_fault():
    w = synth.Workload("bad", B=1, Hq=1, Hkv=1, N=1024, d=128, blk=128, seg=256, mode="topk", density=0.5)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, w.blk, w.seg)
    counts, lists = oracle.select(Q, K, perm, w.blk, w.seg, "topk", density=0.5)
    bad = dict(lists)
    bad[(0, 0, 7)] = np.array([0, 99], np.int32)          # 99 is not a candidate block
    c = counts.copy()
    c[0, 0, 7] = 2
    _, idx_d = pack_lists(c, bad, 4)
    pbs.pbs_attn_fwd(dev(Q), dev(K), dev(V), torch.from_numpy(perm).cuda(), torch.from_numpy(c).cuda(), idx_d,
                     w.blk, w.seg)
    with pytest.raises(pbs.PbsError) as e:
        pbs.pbs_check_device()
    assert e.value.code == -6
    perm2 = perm.copy()
    perm2[0, 0, 5] = 900                                   # leaves its segment
    c2 = np.zeros_like(counts)
    c2[0, 0, 7] = 1
    l2 = {(0, 0, 7): np.array([0], np.int32)}              # block 0 holds logical position 5
    c2_d, idx2_d = pack_lists(c2, l2, 4)
    pbs.pbs_attn_fwd(dev(Q), dev(K), dev(V), torch.from_numpy(perm2).cuda(), c2_d, idx2_d, w.blk, w.seg)
    with pytest.raises(pbs.PbsError):
        pbs.pbs_check_device()
    pbs.pbs_check_device()


def test_head_sharded_runs_match_full_run():
    """One problem split over ranks by KV heads (no collective): running the
    attention on each rank's head slice, passed as strided views, gives
    exactly that slice of the full run."""
    from permuted_block_sparse_b200 import shard
    w = synth.Workload("shard", B=2, Hq=8, Hkv=4, N=2048, d=128, blk=128, seg=512, mode="topk", density=0.2,
                       stripe_frac=0.01)
    Q, K, V, _ = synth.make_inputs(w)
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    perm = pbs.pbs_permute(Qd, Kd, w.blk, w.seg)
    counts, idx = pbs.pbs_select(Qd, Kd, perm, w.blk, w.seg, "topk", w.density)
    O_full, L_full = pbs.pbs_attn_fwd(Qd, Kd, Vd, perm, counts, idx, w.blk, w.seg)
    for rank in range(3):
        lo, hi = shard.kv_head_range(w.Hkv, 3, rank)
        qlo, qhi = shard.query_head_range(w.Hq, w.Hkv, 3, rank)
        O, L = pbs.pbs_attn_fwd(Qd[:, qlo:qhi], Kd[:, lo:hi], Vd[:, lo:hi], perm[:, lo:hi].contiguous(),
                                counts[:, qlo:qhi].contiguous(), idx[:, qlo:qhi].contiguous(), w.blk, w.seg)
        pbs.pbs_check_device()
        assert torch.equal(O, O_full[:, qlo:qhi]), rank
        assert torch.equal(L, L_full[:, qlo:qhi]), rank
