"""Pins for the fp64 oracle: each function is checked against something other
than itself -- brute-force enumeration, closed forms on constructed inputs,
library routines (torch fp64 scaled_dot_product_attention / logsumexp) and
invariants the pages state.

Passages: "Sparser Block-Sparse Attention via Token Permutation" (Technical
Summary 1-4), "S2O: Early Stopping for Sparse Attention via Online
Permutation" (Technical Summary 1-3), "Block Sparse Flash Attention"
(Approach), "SampleAttention" (Technical Deep Dive, cumulative mass).
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from permuted_block_sparse_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _small(B=1, Hq=4, Hkv=2, N=128, d=16, seed=0, scale=1.0):
    Q = synth.random_lattice((B, Hq, N, d), seed, scale)
    K = synth.random_lattice((B, Hkv, N, d), seed + 1, scale)
    V = synth.random_lattice((B, Hkv, N, d), seed + 2, scale)
    return Q, K, V


# ---------------------------------------------------------------------------
# permutation: segmented stable descending sort (PBS Technical Summary 2, 3)
# ---------------------------------------------------------------------------

def _brute_force_segment_order(scores):
    """The unique ordering that is non-increasing in score and ascending in
    position among equal scores, found by enumerating all permutations."""
    n = len(scores)
    found = []
    for p in itertools.permutations(range(n)):
        ok = True
        for a, b in zip(p, p[1:]):
            if scores[a] < scores[b] or (scores[a] == scores[b] and a > b):
                ok = False
                break
        if ok:
            found.append(p)
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_sort_segments_brute_force(seed):
    rng = np.random.default_rng(seed)
    seg, N = 7, 20            # ragged last segment of 6
    scores = rng.integers(-3, 4, size=(1, 2, N)).astype(np.float64)   # many ties
    scores[0, 1, :3] = np.inf                                          # sink-like
    perm = oracle.sort_segments(scores, seg)
    for h in range(2):
        for lo in range(0, N, seg):
            hi = min(lo + seg, N)
            ref = _brute_force_segment_order(list(scores[0, h, lo:hi]))
            assert list(perm[0, h, lo:hi] - lo) == list(ref)


def test_permutation_is_segment_bijection_and_sinks_lead():
    w = synth.WORKLOADS["gqa_8k_band"].with_(N=2048, seg=512)
    Q, K, V, _ = synth.make_inputs(w)
    perm = oracle.permute(Q, K, w.blk, w.seg, n_sink=100)
    for h in range(w.Hkv):
        for lo in range(0, w.N, w.seg):
            assert sorted(perm[0, h, lo:lo + w.seg]) == list(range(lo, lo + w.seg))
        assert list(perm[0, h, :100]) == list(range(100))


def test_proxy_query_closed_form():
    """Earlier query rows are huge noise; the last block of each head of the
    group is a unit vector (e0 for the first head, e1 for the second).  The
    pooled proxy query is then blk*(e0+e1), so keys rank by K[:,0]+K[:,1]."""
    B, Hq, Hkv, N, d, blk, seg = 1, 4, 2, 64, 8, 8, 32
    rng = np.random.default_rng(5)
    Q = np.round(rng.standard_normal((B, Hq, N, d)) * 200).astype(np.float32)
    Q[:, :, N - blk:, :] = 0
    for hk in range(Hkv):
        Q[0, 2 * hk, N - blk:, 0] = 1.0
        Q[0, 2 * hk + 1, N - blk:, 1] = 1.0
    K = synth.random_lattice((B, Hkv, N, d), 6)
    qhat = oracle.proxy_query(Q, Hkv, blk)
    expect = np.zeros(d)
    expect[0] = expect[1] = blk
    for hk in range(Hkv):
        assert np.array_equal(qhat[0, hk], expect)
    perm = oracle.permute(Q, K, blk, seg)
    for hk in range(Hkv):
        key = K[0, hk, :, 0].astype(np.float64) + K[0, hk, :, 1]
        for lo in range(0, N, seg):
            got = key[perm[0, hk, lo:lo + seg]]
            assert np.all(np.diff(got) <= 0)


def test_scores_match_mean_of_attention_logits():
    """The proxy score of key j equals blk*G times the mean, over the pooled
    queries, of the raw logit q.k_j (linearity), computed here from the full
    logit matrix instead of the pooled vector."""
    Q, K, V = _small(N=64, d=16)
    blk = 8
    qhat = oracle.proxy_query(Q, 2, blk)
    s = oracle.key_scores(qhat, K)
    for hk in range(2):
        qs = Q[0, 2 * hk:2 * hk + 2, -blk:, :].reshape(-1, 16).astype(np.float64)
        logits = qs @ K[0, hk].astype(np.float64).T
        assert np.array_equal(s[0, hk], logits.mean(axis=0) * (2 * blk))


# ---------------------------------------------------------------------------
# block selection (PBS Technical Summary 4; SampleAttention cumulative mass)
# ---------------------------------------------------------------------------

def _tile_logit_sum(Q, K, perm, b, hq, i, pb, blk, G):
    hk = hq // G
    q = Q[b, hq, i * blk:(i + 1) * blk].astype(np.float64)
    k = K[b, hk, perm[b, hk, pb * blk:(pb + 1) * blk]].astype(np.float64)
    return (q @ k.T).sum()


def _nat_tile_logit_sum(Q, K, b, hq, i, j, blk, G):
    hk = hq // G
    q = Q[b, hq, i * blk:(i + 1) * blk].astype(np.float64)
    k = K[b, hk, j * blk:(j + 1) * blk].astype(np.float64)
    return (q @ k.T).sum()


def _brute_topk(S, forced, want):
    """Max-sum subset of size ``want`` containing ``forced``; among equal
    sums the lexicographically smallest ascending tuple."""
    n = len(S)
    rest = [x for x in range(n) if x not in forced]
    best = None
    for extra in itertools.combinations(rest, want - len(forced)):
        sub = tuple(sorted(list(forced) + list(extra)))
        val = sum(S[x] for x in sub)
        if best is None or val > best[0] or (val == best[0] and sub < best[1]):
            best = (val, sub)
    return list(best[1])


@pytest.mark.parametrize("density,band,n_sink", [(0.3, 0, 0), (0.45, 0, 8), (0.2, 12, 0), (0.05, 0, 0)])
def test_topk_selection_brute_force(density, band, n_sink):
    B, Hq, Hkv, N, d, blk, seg = 1, 4, 2, 128, 16, 8, 32
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=11)
    perm = oracle.permute(Q, K, blk, seg, n_sink)
    counts, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=density, band=band, n_sink=n_sink)
    G = Hq // Hkv
    spb = seg // blk
    for h in range(Hq):
        inv = oracle.inverse_permutation(perm[0, h // G])
        for i in range(N // blk):
            s = i // spb
            ncand = s * spb
            D = i - s * spb + 1
            if ncand == 0:
                assert counts[0, h, i] == 0
                continue
            S = [_tile_logit_sum(Q, K, perm, 0, h, i, pb, blk, G) for pb in range(ncand)]
            forced = set()
            for pos in range(min(n_sink, s * seg)):
                forced.add(int(inv[pos]) // blk)
            if band:
                for pos in range(max(0, i * blk - band + 1), s * seg):
                    forced.add(int(inv[pos]) // blk)
            k = max(D + len(forced), math.ceil(Fraction(round(density * 1000), 1000) * (i + 1)))
            ref = _brute_topk(S, forced, k - D)
            assert list(lists[(0, h, i)]) == ref, (h, i)


def test_topk_budget_integer_rounding():
    # 0.3 * 10 is 3.0000000000000004 in binary floating point; the budget is 3.
    assert oracle.topk_target(10, 0.3) == 3
    for n in range(1, 300):
        for rho in (0.1, 0.2, 0.3, 0.45, 1.0):
            assert oracle.topk_target(n, rho) == math.ceil(Fraction(round(rho * 1000), 1000) * n)


def _brute_tau(p_diag, p_cand, forced, tau):
    """Smallest set containing ``forced`` whose mass (with the diagonal)
    reaches tau; among those the largest mass, then lexicographic."""
    n = len(p_cand)
    rest = [x for x in range(n) if x not in forced]
    base = sum(p_diag) + sum(p_cand[x] for x in forced)
    for size in range(0, len(rest) + 1):
        best = None
        for extra in itertools.combinations(rest, size):
            mass = base + sum(p_cand[x] for x in extra)
            sub = tuple(sorted(list(forced) + list(extra)))
            if mass >= tau and (best is None or mass > best[0] + 1e-15 or
                                (abs(mass - best[0]) <= 1e-15 and sub < best[1])):
                best = (mass, sub)
        if best is not None:
            return list(best[1])
    return sorted(range(n))


@pytest.mark.parametrize("tau", [0.5, 0.8, 0.95, 0.999])
def test_tau_selection_brute_force(tau):
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 128, 16, 8, 32
    # larger values so block masses differ visibly
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=21, scale=3.0)
    perm = oracle.permute(Q, K, blk, seg)
    counts, lists = oracle.select(Q, K, perm, blk, seg, "tau", tau=tau)
    spb = seg // blk
    for h in range(Hq):
        for i in range(N // blk):
            s = i // spb
            ncand = s * spb
            if ncand == 0:
                continue
            scale = 1.0 / (blk * blk * math.sqrt(d))
            lc = [_tile_logit_sum(Q, K, perm, 0, h, i, pb, blk, 2) * scale for pb in range(ncand)]
            ld = [_nat_tile_logit_sum(Q, K, 0, h, i, j, blk, 2) * scale for j in range(s * spb, i + 1)]
            allv = torch.tensor(lc + ld, dtype=torch.float64)
            p = torch.softmax(allv, 0).numpy()
            ref = _brute_tau(p[ncand:], p[:ncand], set(), tau)
            assert list(lists[(0, h, i)]) == ref, (h, i)


def test_selection_special_cases():
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 128, 16, 8, 32
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=3)
    perm = oracle.permute(Q, K, blk, seg)
    for mode, kw in (("topk", dict(density=1.0)), ("tau", dict(tau=1.0))):
        counts, lists = oracle.select(Q, K, perm, blk, seg, mode, **kw)
        for i in range(N // blk):
            assert list(lists[(0, 0, i)]) == list(range(oracle.n_candidates(i, blk, seg)))
    # one segment spanning everything: no candidates at all (dense diagonal)
    counts, lists = oracle.select(Q, K, oracle.permute(Q, K, blk, N), blk, N, "topk", density=0.1)
    assert counts.sum() == 0
    # tiny density: only forced (none here) -> empty lists
    counts, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=0.001)
    for i in range(N // blk):
        D = i - (i // 4) * 4 + 1
        assert counts[0, 0, i] == max(0, oracle.topk_target(i + 1, 0.001) - D)


# ---------------------------------------------------------------------------
# attention (S2O Technical Summary 3; PBS Technical Summary 1)
# ---------------------------------------------------------------------------

def _sdpa(q, k, v, mask=None, causal=False):
    q = torch.from_numpy(q.astype(np.float64))
    k = torch.from_numpy(k.astype(np.float64))
    v = torch.from_numpy(v.astype(np.float64))
    m = None if mask is None else torch.from_numpy(mask)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m, is_causal=causal).numpy()


def test_dense_equals_textbook_causal_attention():
    B, Hq, Hkv, N, d, blk, seg = 2, 4, 2, 128, 16, 16, 32
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=7)
    perm = oracle.permute(Q, K, blk, seg)
    _, lists = oracle.dense_lists(B, Hq, N // blk, blk, seg)
    O, L = oracle.attn(Q, K, V, perm, lists, blk, seg)
    G = Hq // Hkv
    Kr = np.repeat(K, G, axis=1)
    Vr = np.repeat(V, G, axis=1)
    ref = _sdpa(Q, Kr, Vr, causal=True)
    assert np.max(np.abs(O - ref)) < 1e-12
    logits = torch.from_numpy(Q.astype(np.float64)) @ torch.from_numpy(Kr.astype(np.float64)).transpose(-1, -2) / math.sqrt(d)
    logits = logits.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), -math.inf)
    assert np.max(np.abs(L - torch.logsumexp(logits, -1).numpy())) < 1e-12


def _explicit_mask(N, blk, seg, perm_row, lists_h):
    """Boolean [N, N] mask built position by position from the lists."""
    mask = np.zeros((N, N), bool)
    for q in range(N):
        i = q // blk
        s_start = (i * blk // seg) * seg
        for k in range(s_start, q + 1):
            mask[q, k] = True
        for pb in lists_h.get(i, []):
            for r in range(blk):
                mask[q, perm_row[pb * blk + r]] = True
    return mask


@pytest.mark.parametrize("mode,kw", [("topk", dict(density=0.3)), ("tau", dict(tau=0.9)),
                                     ("topk", dict(density=0.2, band=20, n_sink=5))])
def test_sparse_attention_equals_masked_sdpa(mode, kw):
    B, Hq, Hkv, N, d, blk, seg = 1, 4, 2, 128, 16, 8, 32
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=8, scale=2.0)
    perm = oracle.permute(Q, K, blk, seg, kw.get("n_sink", 0))
    counts, lists = oracle.select(Q, K, perm, blk, seg, mode, **kw)
    O, L = oracle.attn(Q, K, V, perm, lists, blk, seg)
    G = Hq // Hkv
    for h in range(Hq):
        lh = {i: list(lists[(0, h, i)]) for i in range(N // blk)}
        mask = _explicit_mask(N, blk, seg, perm[0, h // G], lh)
        assert not np.any(np.triu(mask, 1)), "future key in the key set"
        ref = _sdpa(Q[0, h], K[0, h // G], V[0, h // G], mask=mask)
        assert np.max(np.abs(O[0, h] - ref)) < 1e-12


def test_zero_weight_on_future_tokens():
    """Explicit attention weights: a future key never gets weight, and the
    output of a row does not change when every future K/V row is replaced
    by large values."""
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 64, 8, 8, 16
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=9)
    perm = oracle.permute(Q, K, blk, seg)
    counts, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=0.5)
    O, _ = oracle.attn(Q, K, V, perm, lists, blk, seg)
    for cut in (20, 33, 47):
        K2, V2 = K.copy(), V.copy()
        K2[:, :, cut:] = 31.875
        V2[:, :, cut:] = -31.875
        O2, _ = oracle.attn(Q, K2, V2, perm, lists, blk, seg)
        assert np.array_equal(O[:, :, :cut], O2[:, :, :cut])


def test_joint_kv_permutation_invariance():
    """Attention depends on the key set, not on where the rows sit: moving
    K/V rows of earlier segments by a permutation sigma and composing the
    index list with sigma^-1 leaves every output of the last segment
    unchanged; so does visiting the listed blocks in another order."""
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 128, 16, 8, 32
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=10)
    perm = oracle.permute(Q, K, blk, seg)
    counts, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=0.4)
    rng = np.random.default_rng(0)
    sigma = np.arange(N)
    for lo in range(0, N - seg, seg):           # last segment stays in place
        sigma[lo:lo + seg] = lo + rng.permutation(seg)
    inv_sigma = np.empty_like(sigma)
    inv_sigma[sigma] = np.arange(N)
    K2 = K[:, :, sigma]
    V2 = V[:, :, sigma]
    perm2 = inv_sigma[perm].astype(np.int32)
    last = [(0, h, i) for h in range(Hq) for i in range((N - seg) // blk, N // blk)]
    O1, L1 = oracle.attn(Q, K, V, perm, lists, blk, seg, blocks=last)
    O2, L2 = oracle.attn(Q, K2, V2, perm2, lists, blk, seg, blocks=last)
    sl = slice(N - seg, N)
    assert np.max(np.abs(O1[:, :, sl] - O2[:, :, sl])) < 1e-12
    shuffled = {key: rng.permutation(v) for key, v in lists.items()}
    O3, _ = oracle.attn(Q, K, V, perm, shuffled, blk, seg, blocks=last)
    assert np.max(np.abs(O1[:, :, sl] - O3[:, :, sl])) < 1e-12


# ---------------------------------------------------------------------------
# gating (Block Sparse Flash Attention, Approach)
# ---------------------------------------------------------------------------

def _brute_tile_max(q, k, qpos, kpos):
    best = -math.inf
    for a in range(q.shape[0]):
        for c in range(k.shape[0]):
            if kpos[c] <= qpos[a]:
                v = float(np.dot(q[a].astype(np.float64), k[c].astype(np.float64)))
                best = max(best, v)
    return best


def test_gate_brute_force_and_reduction():
    B, Hq, Hkv, N, d, blk = 1, 2, 1, 64, 8, 8
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=12, scale=2.0)
    seg = blk
    perm = np.broadcast_to(np.arange(N, dtype=np.int32), (B, Hkv, N)).copy()
    counts, lists = oracle.dense_lists(B, Hq, N // blk, blk, seg)
    keep = 3
    thr = oracle.calibrate_thresholds(Q, K, blk, keep)
    # thr = -inf reduces to the ungated result
    O0, _ = oracle.attn(Q, K, V, perm, lists, blk, seg)
    Oinf, _ = oracle.attn(Q, K, V, perm, lists, blk, seg, gate_thr=np.full_like(thr, -np.inf))
    assert np.array_equal(O0, Oinf)
    Og, _ = oracle.attn(Q, K, V, perm, lists, blk, seg, gate_thr=thr)
    for h in range(Hq):
        mask = np.zeros((N, N), bool)
        for i in range(N // blk):
            qpos = np.arange(i * blk, (i + 1) * blk)
            M = []
            for j in range(i + 1):
                kpos = np.arange(j * blk, (j + 1) * blk)
                M.append(_brute_tile_max(Q[0, h, qpos], K[0, 0, kpos], qpos, kpos))
            t = -math.inf if i + 1 <= keep else sorted(M, reverse=True)[keep - 1]
            assert t == thr[0, h, i]
            for j in range(i + 1):
                if j == i or M[j] >= t:
                    for a in qpos:
                        for c in range(j * blk, (j + 1) * blk):
                            mask[a, c] = c <= a
        ref = _sdpa(Q[0, h], K[0, 0], V[0, 0], mask=mask)
        assert np.max(np.abs(Og[0, h] - ref)) < 1e-12


# ---------------------------------------------------------------------------
# synthetic inputs
# ---------------------------------------------------------------------------

def test_inputs_are_bf16_exact_lattice():
    w = synth.WORKLOADS["single_head_1k"]
    Q, K, V, info = synth.make_inputs(w)
    for X in (Q, K, V):
        assert np.all(X * 8 == np.round(X * 8))
        assert np.abs(X).max() <= 31.875
        t = torch.from_numpy(X).to(torch.bfloat16).to(torch.float32).numpy()
        assert np.array_equal(t, X)
    assert info["stripes"].shape == (1, 1, 20)
    Q2, K2, V2, _ = synth.make_inputs(w)
    assert np.array_equal(Q, Q2) and np.array_equal(K, K2)


def test_local_window_recipe():
    """The planted local window draws no random numbers (without it the
    same seed gives the same Q and K as before, up to the positional
    vector), keeps values bf16-exact, and raises q.k near the diagonal."""
    base = synth.WORKLOADS["sample_32k_local"].with_(N=2048, seg=512, Hq=4, Hkv=1)
    Q, K, V, _ = synth.make_inputs(base)
    Q0, K0, V0, _ = synth.make_inputs(base.with_(local_amp=0.0))
    assert np.array_equal(V, V0)                     # V never gets the positional vector
    for X in (Q, K):
        assert np.all(X * 8 == np.round(X * 8)) and np.abs(X).max() <= 31.875
    lg = Q[0, 0].astype(np.float64) @ K[0, 0].astype(np.float64).T
    n = np.arange(base.N)
    near = np.abs(n[:, None] - n[None, :]) < 8
    far = np.abs(n[:, None] - n[None, :]) > 512
    assert lg[near].mean() > lg[far].mean() + 50.0
    lg0 = Q0[0, 0].astype(np.float64) @ K0[0, 0].astype(np.float64).T
    assert abs(lg0[near].mean() - lg0[far].mean()) < 5.0


def test_stripe_keys_cluster_in_leading_blocks():
    """With planted stripes, the permutation must gather the stripe keys into
    the first permuted block of their segment (the clustering the method is
    after).  A random key can outscore a stripe key by chance, so the check
    is on the fraction, not on every key."""
    w = synth.WORKLOADS["single_head_1k"]
    Q, K, V, info = synth.make_inputs(w)
    perm = oracle.permute(Q, K, w.blk, w.seg)
    inv = oracle.inverse_permutation(perm[0, 0])
    rel = inv[info["stripes"][0, 0]] % w.seg
    assert np.mean(rel < w.blk) >= 0.95
    # without the permutation the stripes sit wherever they were drawn
    assert np.mean(info["stripes"][0, 0] % w.seg < w.blk) < 0.5


# ---------------------------------------------------------------------------
# S2O visiting order and early stopping ("S2O: Early Stopping for Sparse
# Attention via Online Permutation", Technical Summary 2 and 3)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode,kw", [("topk", dict(density=0.4, n_sink=8)), ("tau", dict(tau=0.9)),
                                     ("topk", dict(density=1.0))])
def test_score_order_lists(mode, kw):
    """Score order holds the same set as the ascending list; sink-forced
    blocks lead in ascending order; the rest is non-increasing in the block
    score (recomputed here as a sum of explicit logits), ties ascending."""
    B, Hq, Hkv, N, d, blk, seg = 1, 4, 2, 128, 16, 8, 32
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=31)
    n_sink = kw.get("n_sink", 0)
    perm = oracle.permute(Q, K, blk, seg, n_sink)
    c_a, l_a = oracle.select(Q, K, perm, blk, seg, mode, **kw)
    c_s, l_s = oracle.select(Q, K, perm, blk, seg, mode, list_order="score", **kw)
    assert np.array_equal(c_a, c_s)
    G = Hq // Hkv
    spb = seg // blk
    checked = 0
    for (b, h, i), arr in l_s.items():
        assert sorted(arr.tolist()) == l_a[(b, h, i)].tolist()
        if arr.size < 2:
            continue
        inv = oracle.inverse_permutation(perm[0, h // G])
        s = i // spb
        forced = {int(inv[pos]) // blk for pos in range(min(n_sink, s * seg))}
        nf = sum(1 for x in arr.tolist() if x in forced)
        assert set(arr[:nf].tolist()) == forced
        assert arr[:nf].tolist() == sorted(arr[:nf].tolist())
        S = [_tile_logit_sum(Q, K, perm, 0, h, i, int(pb), blk, G) for pb in arr[nf:]]
        for (s1, a1), (s2, a2) in zip(zip(S, arr[nf:]), zip(S[1:], arr[nf + 1:])):
            assert s1 > s2 or (s1 == s2 and a1 < a2), (h, i)
        checked += 1
    assert checked > 10


def _es_case(seed=41):
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 512, 16, 16, 128
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=seed, scale=2.0)
    perm = oracle.permute(Q, K, blk, seg)
    _, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=1.0, list_order="score")
    return blk, seg, d, Q, K, V, perm, lists


def _explicit_gains(Q, K, perm, h, i, listed, blk, seg, scale):
    """Per Pass-2 tile k: max over the block's rows of (exp mass of tile k) /
    (exp mass of the own segment's visible keys and tiles 1..k), from
    explicit exponentials of the logits (no running state)."""
    rows = np.arange(i * blk, (i + 1) * blk)
    q = Q[0, h, rows].astype(np.float64)
    s0 = (i // (seg // blk)) * seg
    own = np.arange(s0, (i + 1) * blk)
    lo = (q @ K[0, 0, own].astype(np.float64).T) * scale
    total = np.where(own[None, :] <= rows[:, None], np.exp(lo), 0.0).sum(axis=1)
    gains = []
    for pb in listed:
        pos = perm[0, 0, int(pb) * blk:(int(pb) + 1) * blk]
        et = np.exp((q @ K[0, 0, pos].astype(np.float64).T) * scale).sum(axis=1)
        total = total + et
        gains.append(float((et / total).max()))
    return gains


def test_early_stop_brute_force():
    """The early-stopped result equals plain masked attention over the own
    segment and the first k* listed blocks, where k* is the first tile whose
    explicit mass ratio is below tau (all of them if none is)."""
    blk, seg, d, Q, K, V, perm, lists = _es_case()
    scale = 1.0 / math.sqrt(d)
    n_mid = 0
    for (b, h, i), listed in lists.items():
        if listed.size < 3:
            continue
        gains = _explicit_gains(Q, K, perm, h, i, listed, blk, seg, scale)
        for tau in (float(np.median(gains)), float(np.min(gains)) * 1.0001, float(np.max(gains)) * 0.999):
            k_star = next((k + 1 for k, g in enumerate(gains) if g < tau), len(gains))
            O, L, n = oracle.attn_early_stop_block(Q, K, V, perm, listed, b, h, i, blk, seg, scale, tau)
            O_ref, L_ref = oracle.attn_block(Q, K, V, perm, listed[:k_star], b, h, i, blk, seg, scale)
            assert n == k_star, (h, i, tau)
            np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
            np.testing.assert_allclose(L, L_ref, rtol=0, atol=1e-12)
            n_mid += 0 < k_star < len(gains)
    assert n_mid > 5


def test_early_stop_limits():
    """tau = 0 never stops (plain sparse attention over every listed block);
    tau > 1 stops right after the first listed block (a gain is at most 1)."""
    blk, seg, d, Q, K, V, perm, lists = _es_case(seed=43)
    scale = 1.0 / math.sqrt(d)
    for (b, h, i), listed in lists.items():
        O, L, n = oracle.attn_early_stop_block(Q, K, V, perm, listed, b, h, i, blk, seg, scale, 0.0)
        O_ref, L_ref = oracle.attn_block(Q, K, V, perm, listed, b, h, i, blk, seg, scale)
        assert n == len(listed)
        np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
        O, L, n = oracle.attn_early_stop_block(Q, K, V, perm, listed, b, h, i, blk, seg, scale, 1.5)
        O_ref, L_ref = oracle.attn_block(Q, K, V, perm, listed[:1], b, h, i, blk, seg, scale)
        assert n == min(1, len(listed))
        np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# attention coverage (PBS page, Key Results)
# ---------------------------------------------------------------------------

def test_coverage_definition():
    """Coverage is 1 with every candidate listed; with a partial list it
    equals exp(LSE over the key set - LSE over all causal keys), the two
    LSEs taken from the (SDPA-pinned) attention oracle; it never decreases
    as blocks are added."""
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 512, 16, 16, 128
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=51, scale=2.0)
    perm = oracle.permute(Q, K, blk, seg)
    scale = 1.0 / math.sqrt(d)
    _, full = oracle.select(Q, K, perm, blk, seg, "topk", density=1.0)
    _, part = oracle.select(Q, K, perm, blk, seg, "topk", density=0.3, list_order="score")
    checked = 0
    for (b, h, i), listed in part.items():
        c_full = oracle.coverage_block(Q, K, perm, full[(b, h, i)], b, h, i, blk, seg, scale)
        np.testing.assert_allclose(c_full, 1.0, rtol=0, atol=1e-12)
        c = oracle.coverage_block(Q, K, perm, listed, b, h, i, blk, seg, scale)
        _, l_sel = oracle.attn_block(Q, K, V, perm, listed, b, h, i, blk, seg, scale)
        _, l_all = oracle.attn_block(Q, K, V, perm, full[(b, h, i)], b, h, i, blk, seg, scale)
        np.testing.assert_allclose(c, np.exp(l_sel - l_all), rtol=1e-12, atol=0)
        prev = oracle.coverage_block(Q, K, perm, listed[:0], b, h, i, blk, seg, scale)
        for k in range(1, len(listed) + 1):
            cur = oracle.coverage_block(Q, K, perm, listed[:k], b, h, i, blk, seg, scale)
            assert np.all(cur >= prev - 1e-15)
            prev = cur
        checked += len(listed) > 0
    assert checked > 10


# ---------------------------------------------------------------------------
# per-query-segment key permutation (S2O, Technical Summary 1: historical
# KV permutation, one ranking of the earlier keys per query segment)
# ---------------------------------------------------------------------------

def test_segment_queries_closed_form():
    """The representative query of segment s is the plain sum of its rows
    over the group's heads: checked on inputs whose rows encode their
    position, head and dimension."""
    B, Hq, Hkv, N, d, seg = 1, 4, 2, 64, 8, 16
    Q = np.zeros((B, Hq, N, d), np.float32)
    for h in range(Hq):
        for n in range(N):
            Q[0, h, n] = (h + 1) * 0.125 + (n % seg) * 0.5 + np.arange(d) * 0.25 + (n // seg) * 4
    qs = oracle.segment_queries(Q, Hkv, seg)
    G = Hq // Hkv
    for hk in range(Hkv):
        for s in range(N // seg):
            # closed form: sum over heads g and rows r of the formula above
            heads = sum((hk * G + g + 1) * 0.125 for g in range(G)) * seg
            rows = G * sum(r * 0.5 for r in range(seg))
            want = heads + rows + G * seg * (np.arange(d) * 0.25 + s * 4)
            np.testing.assert_allclose(qs[0, hk, s], want, rtol=0, atol=1e-9)


@pytest.mark.parametrize("seed", [0, 1])
def test_permute_segmented_brute_force(seed):
    """Per query segment s: every key segment before s is the unique stable
    descending order of its keys' scores against s's representative query
    (brute-force enumeration); key segments from s on keep natural order."""
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 32, 4, 2, 8
    Q = synth.random_lattice((B, Hq, N, d), seed, 1.0)
    K = synth.random_lattice((B, Hkv, N, d), seed + 5, 1.0)
    K[0, 0, 3] = K[0, 0, 5]                          # a tie inside key segment 0
    perm = oracle.permute_segmented(Q, K, blk, seg)
    for s in range(N // seg):
        qs = Q[0, :, s * seg:(s + 1) * seg].astype(np.float64).reshape(-1, d).sum(axis=0)
        for j in range(N // seg):
            got = perm[0, 0, s, j * seg:(j + 1) * seg]
            if j >= s:
                assert got.tolist() == list(range(j * seg, (j + 1) * seg))
                continue
            sc = [float(K[0, 0, j * seg + x].astype(np.float64) @ qs) for x in range(seg)]
            ref = _brute_force_segment_order(sc)
            assert got.tolist() == [j * seg + x for x in ref], (s, j)


def test_segmented_permutation_reduces_to_shared_one():
    """When every segment has the same representative query, each query
    segment's permutation of its prefix equals the shared permutation
    sorted by that query."""
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 64, 8, 8, 16
    Q = np.zeros((B, Hq, N, d), np.float32)
    base = synth.random_lattice((B, Hq, seg, d), 3, 1.0)
    for s in range(N // seg):
        Q[:, :, s * seg:(s + 1) * seg] = base
    K = synth.random_lattice((B, Hkv, N, d), 4, 1.0)
    perm = oracle.permute_segmented(Q, K, blk, seg)
    qs = oracle.segment_queries(Q, Hkv, seg)[:, :, 0]
    shared = oracle.sort_segments(oracle.key_scores(qs, K), seg)
    for s in range(N // seg):
        assert np.array_equal(perm[0, 0, s, :s * seg], shared[0, 0, :s * seg])


@pytest.mark.parametrize("mode,kw", [("topk", dict(density=0.3)), ("tau", dict(tau=0.9)),
                                     ("topk", dict(density=0.2, band=20, n_sink=5))])
def test_segmented_sparse_attention_equals_masked_sdpa(mode, kw):
    """With one permutation per query segment, every block's key set (built
    position by position from its segment's permutation) gives the same O
    as torch fp64 SDPA under that mask; stacking one shared permutation for
    every segment reproduces the shared-permutation selection exactly."""
    B, Hq, Hkv, N, d, blk, seg = 1, 4, 2, 128, 16, 8, 32
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=9, scale=2.0)
    n_sink = kw.get("n_sink", 0)
    perm4 = oracle.permute_segmented(Q, K, blk, seg, n_sink)
    counts, lists = oracle.select(Q, K, perm4, blk, seg, mode, **kw)
    O, L = oracle.attn(Q, K, V, perm4, lists, blk, seg)
    G = Hq // Hkv
    for h in range(Hq):
        mask = np.zeros((N, N), bool)
        for q in range(N):
            i = q // blk
            s = i * blk // seg
            mask[q, s * seg:q + 1] = True
            for pb in lists[(0, h, i)]:
                mask[q, perm4[0, h // G, s, pb * blk:(pb + 1) * blk]] = True
        assert not np.any(np.triu(mask, 1))
        ref = _sdpa(Q[0, h], K[0, h // G], V[0, h // G], mask=mask)
        assert np.max(np.abs(O[0, h] - ref)) < 1e-12
    perm3 = oracle.permute(Q, K, blk, seg, n_sink)
    stacked = np.repeat(perm3[:, :, None, :], N // seg, axis=2)
    c3, l3 = oracle.select(Q, K, perm3, blk, seg, mode, **kw)
    c4, l4 = oracle.select(Q, K, stacked, blk, seg, mode, **kw)
    assert np.array_equal(c3, c4)
    assert all(np.array_equal(l3[k], l4[k]) for k in l3)


# ---------------------------------------------------------------------------
# SampleAttention-style selector ("SampleAttention", Technical Deep Dive,
# Stage 1 Trunk Sampling and Stage 2 Score-Based Filtering)
# ---------------------------------------------------------------------------

def test_sample_pattern_scores_explicit():
    """Column and slash scores equal sums over an explicit torch fp64 softmax
    of the sampled rows (the last block of every segment)."""
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 96, 8, 8, 32
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=61, scale=2.0)
    scale = 1.0 / math.sqrt(d)
    rows = oracle.sample_trunk_rows(N, blk, seg)
    assert rows.tolist() == [r for s in range(N // seg) for r in range(s * seg + seg - blk, (s + 1) * seg)]
    for h in range(Hq):
        col, sl = oracle.sample_pattern_scores(Q, K, 0, h, blk, seg, scale)
        lg = torch.from_numpy(Q[0, h].astype(np.float64)) @ torch.from_numpy(K[0, 0].astype(np.float64)).T * scale
        mask = torch.tril(torch.ones(N, N, dtype=torch.bool))
        P = torch.softmax(lg.masked_fill(~mask, float("-inf")), dim=1).numpy()
        want_col = P[rows].sum(axis=0)
        want_sl = np.zeros(N)
        for q in rows:
            for k in range(q + 1):
                want_sl[q - k] += P[q, k]
        np.testing.assert_allclose(col, want_col, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(sl, want_sl, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("alpha", [0.3, 0.6, 0.9, 0.99])
def test_cumulative_cut_is_smallest_set(alpha):
    rng = np.random.default_rng(5)
    for _ in range(20):
        sc = rng.random(9) ** 3
        keep = oracle.cumulative_cut(sc, alpha)
        goal = alpha * sc.sum()
        assert sc[keep].sum() >= goal
        best = None
        for size in range(0, 10):
            if any(sum(sc[list(c)]) >= goal for c in itertools.combinations(range(9), size)):
                best = size
                break
        assert keep.sum() == best
        # the kept entries are the highest scores
        assert sc[keep].min() >= sc[~keep].max() if (~keep).any() else True
    assert oracle.cumulative_cut(np.array([0.5, 0.0, 0.2]), 1.0).tolist() == [True, False, True]


@pytest.mark.parametrize("alpha", [0.5, 0.9, 1.0])
def test_select_sample_matches_position_mask(alpha):
    """Block lists equal the blocks touched by the position-level pattern
    mask kept_column[k] or kept_slash[q - k], restricted to earlier
    segments; alpha = 1 lists every candidate."""
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 128, 16, 8, 32
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=62, scale=2.0)
    scale = 1.0 / math.sqrt(d)
    counts, lists = oracle.select_sample(Q, K, blk, seg, alpha)
    for h in range(Hq):
        col, sl = oracle.sample_pattern_scores(Q, K, 0, h, blk, seg, scale)
        kc, ks = oracle.cumulative_cut(col, alpha), oracle.cumulative_cut(sl, alpha)
        for i in range(N // blk):
            ncand = oracle.n_candidates(i, blk, seg)
            want = set()
            for q in range(i * blk, (i + 1) * blk):
                for k in range(ncand * blk):
                    if k <= q and (kc[k] or ks[q - k]):
                        want.add(k // blk)
            assert lists[(0, h, i)].tolist() == sorted(want), (h, i)
            if alpha >= 1.0:
                assert lists[(0, h, i)].tolist() == list(range(ncand))


def test_select_sample_lists_grow_with_alpha():
    """Each family's cut keeps the highest scores up to the target, so a
    larger target keeps a superset of columns and offsets, and every block
    list at a smaller target is contained in the list at a larger one."""
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 256, 16, 16, 64
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=71, scale=2.0)
    prev = None
    for alpha in (0.2, 0.5, 0.8, 0.95, 1.0):
        _, lists = oracle.select_sample(Q, K, blk, seg, alpha)
        if prev is not None:
            for key, arr in lists.items():
                assert set(prev[key].tolist()) <= set(arr.tolist()), (alpha, key)
        prev = lists


def test_select_sample_single_sink_column():
    """All attention on key 0 (a sink): a key aligned with every query at a
    logit of about 34 against 0 elsewhere.  Every trunk row puts more than
    1 - 1e-12 of its mass on key 0, so the column cut keeps key 0 alone for
    any target up to 0.99, and every query block past the first segment
    lists block 0 (the first segment has no candidates)."""
    N, d, blk, seg = 128, 8, 16, 32
    Q = np.zeros((1, 1, N, d), np.float32)
    K = np.zeros((1, 1, N, d), np.float32)
    Q[..., 0] = 4.0
    K[0, 0, 0, 0] = 24.0                         # logit 96 / sqrt(8) ~ 33.9 against 0 elsewhere
    scale = 1.0 / math.sqrt(d)
    col, sl = oracle.sample_pattern_scores(Q, K, 0, 0, blk, seg, scale)
    rows = oracle.sample_trunk_rows(N, blk, seg)
    assert col[0] > len(rows) * (1 - 1e-12)
    for alpha in (0.3, 0.9, 0.99):
        kc = oracle.cumulative_cut(col, alpha)
        assert np.flatnonzero(kc).tolist() == [0]
    counts, lists = oracle.select_sample(Q, K, blk, seg, 0.5)
    for i in range(N // blk):
        if oracle.n_candidates(i, blk, seg) > 0:
            assert 0 in lists[(0, 0, i)].tolist(), i
        else:
            assert lists[(0, 0, i)].size == 0


# ---------------------------------------------------------------------------
# S2O query permutation (Technical Summary 1: Query Permutation); oracle
# only, no GPU path yet
# ---------------------------------------------------------------------------

def test_permute_queries_orders_by_summed_logits():
    """Within each segment the queries come in descending order of the sum
    of their logits over all keys (explicit Q K^T row sums), equal sums in
    ascending position; each segment maps onto itself."""
    B, Hq, Hkv, N, d, seg = 1, 4, 2, 64, 8, 16
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=81, scale=2.0)
    K[0, 0, :, :] = np.round(K[0, 0, :, :])                  # encourage exact ties
    qperm = oracle.permute_queries(Q, K, seg)
    G = Hq // Hkv
    for h in range(Hq):
        lg = Q[0, h].astype(np.float64) @ K[0, h // G].astype(np.float64).T
        rowsum = lg.sum(axis=1)
        for lo in range(0, N, seg):
            p = qperm[0, h, lo:lo + seg]
            assert sorted(p.tolist()) == list(range(lo, lo + seg))
            sc = rowsum[p]
            for a in range(seg - 1):
                assert sc[a] > sc[a + 1] or (sc[a] == sc[a + 1] and p[a] < p[a + 1]), (h, lo, a)


def test_attn_qperm_identity_is_natural_attention():
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 128, 16, 16, 32
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=82)
    perm = oracle.permute(Q, K, blk, seg)
    _, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=0.4)
    ident = np.broadcast_to(np.arange(N, dtype=np.int32), (B, Hq, N)).copy()
    O1, L1 = oracle.attn_qperm(Q, K, V, perm, ident, lists, blk, seg)
    O2, L2 = oracle.attn(Q, K, V, perm, lists, blk, seg)
    assert np.max(np.abs(O1 - O2)) < 1e-12 and np.max(np.abs(L1 - L2)) < 1e-12


def test_attn_qperm_matches_position_mask():
    """With permuted queries, row q (in permuted block i) sees its own
    segment up to q and the keys of block i's listed permuted blocks: equal to
    torch SDPA with that mask built position by position."""
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 128, 16, 16, 64
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=83, scale=1.5)
    perm = oracle.permute(Q, K, blk, seg)
    qperm = oracle.permute_queries(Q, K, seg)
    Qp = oracle.gather_queries(Q, qperm)
    _, lists = oracle.select(Qp, K, perm, blk, seg, "topk", density=0.3)
    O, L = oracle.attn_qperm(Q, K, V, perm, qperm, lists, blk, seg)
    for h in range(Hq):
        inv = np.empty(N, np.int64)
        inv[qperm[0, h]] = np.arange(N)
        mask = np.zeros((N, N), bool)
        for q in range(N):
            i = inv[q] // blk
            s0 = (q // seg) * seg
            mask[q, s0:q + 1] = True
            for pb in lists.get((0, h, i), []):
                mask[q, perm[0, 0, pb * blk:(pb + 1) * blk]] = True
        ref = _sdpa(Q[0, h][None], K[0, 0][None], V[0, 0][None], mask=mask[None])[0]
        assert np.max(np.abs(O[0, h] - ref)) < 1e-12, h


def test_attn_qperm_dense_lists_give_causal_attention():
    """Listing every candidate makes each row's key set its whole causal
    prefix, whatever the query order."""
    B, Hq, Hkv, N, d, blk, seg = 1, 2, 1, 128, 16, 16, 32
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=84)
    perm = oracle.permute(Q, K, blk, seg)
    qperm = oracle.permute_queries(Q, K, seg)
    _, lists = oracle.dense_lists(B, Hq, N // blk, blk, seg)
    O, L = oracle.attn_qperm(Q, K, V, perm, qperm, lists, blk, seg)
    ref = _sdpa(Q, np.repeat(K, Hq // Hkv, axis=1), np.repeat(V, Hq // Hkv, axis=1), causal=True)
    assert np.max(np.abs(O - ref)) < 1e-12


# ---------------------------------------------------------------------------
# property-based variants of the brute-force pins (random shapes and seeds)
# ---------------------------------------------------------------------------

from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(seed=st.integers(0, 10_000), G=st.sampled_from([1, 2]), blk=st.sampled_from([4, 8]),
       spb=st.sampled_from([2, 3]), nseg=st.sampled_from([2, 3, 4]), density=st.sampled_from([0.1, 0.25, 0.5]),
       n_sink=st.sampled_from([0, 4]))
def test_topk_selection_brute_force_random(seed, G, blk, spb, nseg, density, n_sink):
    d, Hkv = 8, 1
    seg = blk * spb
    N = seg * nseg
    Q, K, V = _small(1, G * Hkv, Hkv, N, d, seed=seed, scale=2.0)
    perm = oracle.permute(Q, K, blk, seg, n_sink)
    counts, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=density, n_sink=n_sink)
    for h in range(G):
        inv = oracle.inverse_permutation(perm[0, 0])
        for i in range(N // blk):
            s = i // spb
            ncand, D = s * spb, i - s * spb + 1
            if ncand == 0:
                assert counts[0, h, i] == 0
                continue
            S = [_tile_logit_sum(Q, K, perm, 0, h, i, pb, blk, G) for pb in range(ncand)]
            forced = {int(inv[pos]) // blk for pos in range(min(n_sink, s * seg))}
            k = max(D + len(forced), math.ceil(Fraction(round(density * 1000), 1000) * (i + 1)))
            k = min(k, D + ncand)
            assert list(lists[(0, h, i)]) == _brute_topk(S, forced, k - D), (h, i)


@settings(max_examples=20, deadline=None)
@given(seed=st.integers(0, 10_000), blk=st.sampled_from([4, 8]), spb=st.sampled_from([2, 4]),
       nseg=st.sampled_from([2, 3]), keep=st.floats(0.0, 1.0))
def test_attention_matches_position_mask_random(seed, blk, spb, nseg, keep):
    """Any lists of candidate blocks: the oracle equals torch fp64 SDPA with
    the key set built position by position (own segment causal, plus the
    listed permuted blocks' keys)."""
    d, seg = 8, blk * spb
    N = seg * nseg
    Q, K, V = _small(1, 1, 1, N, d, seed=seed, scale=1.5)
    perm = oracle.permute(Q, K, blk, seg)
    rng = np.random.default_rng(seed)
    lists = {}
    for i in range(N // blk):
        ncand = (i // spb) * spb
        chosen = [pb for pb in range(ncand) if rng.random() < keep]
        lists[(0, 0, i)] = np.array(chosen, np.int32)
    O, L = oracle.attn(Q, K, V, perm, lists, blk, seg)
    mask = np.zeros((N, N), bool)
    for q in range(N):
        i, s0 = q // blk, (q // seg) * seg
        mask[q, s0:q + 1] = True
        for pb in lists[(0, 0, i)]:
            mask[q, perm[0, 0, pb * blk:(pb + 1) * blk]] = True
    ref = _sdpa(Q[0, 0][None], K[0, 0][None], V[0, 0][None], mask=mask[None])[0]
    assert np.max(np.abs(O[0, 0] - ref)) < 1e-12


@settings(max_examples=40, deadline=None)
@given(seed=st.integers(0, 10_000), n=st.integers(1, 9), alpha=st.floats(0.01, 0.999),
       ties=st.booleans())
def test_cumulative_cut_random(seed, n, alpha, ties):
    """The cut is a smallest set of entries reaching alpha of the total, made
    of the highest scores, equal scores taken in ascending index."""
    rng = np.random.default_rng(seed)
    sc = rng.random(n)
    if ties:
        sc = np.round(sc * 3) / 3                      # repeated values
    if sc.sum() == 0:
        sc[0] = 1.0
    keep = oracle.cumulative_cut(sc, alpha)
    goal = alpha * sc.sum()
    assert sc[keep].sum() >= goal - 1e-12
    smallest = next(size for size in range(n + 1)
                    if any(sum(sc[list(c)]) >= goal for c in itertools.combinations(range(n), size)))
    assert keep.sum() == smallest
    order = sorted(range(n), key=lambda x: (-sc[x], x))
    assert np.flatnonzero(keep).tolist() == sorted(order[:smallest])


@settings(max_examples=25, deadline=None)
@given(seed=st.integers(0, 10_000), seg=st.sampled_from([3, 5, 8]), nseg=st.integers(1, 3),
       ties=st.booleans())
def test_sort_segments_random(seed, seg, nseg, ties):
    rng = np.random.default_rng(seed)
    N = seg * nseg - (seed % seg if nseg > 1 else 0)          # ragged last segment
    sc = rng.standard_normal((1, 1, N))
    if ties:
        sc = np.round(sc)
    perm = oracle.sort_segments(sc, seg)
    for lo in range(0, N, seg):
        hi = min(lo + seg, N)
        assert perm[0, 0, lo:hi].tolist() == [lo + x for x in _brute_force_segment_order(list(sc[0, 0, lo:hi]))]


@settings(max_examples=20, deadline=None)
@given(seed=st.integers(0, 10_000), tau_q=st.floats(0.05, 0.95))
def test_early_stop_brute_force_random(seed, tau_q):
    """Random inputs and a threshold at a random quantile of the explicit
    gains: the early-stopped block equals masked attention over the prefix
    of the visiting order that ends at the first tile below the threshold."""
    blk, seg, d = 8, 32, 8
    Q, K, V = _small(1, 1, 1, 160, d, seed=seed, scale=2.0)
    perm = oracle.permute(Q, K, blk, seg)
    _, lists = oracle.select(Q, K, perm, blk, seg, "topk", density=1.0, list_order="score")
    scale = 1.0 / math.sqrt(d)
    for (b, h, i), listed in lists.items():
        if listed.size < 2:
            continue
        gains = _explicit_gains(Q, K, perm, h, i, listed, blk, seg, scale)
        tau = float(np.quantile(gains, tau_q))
        if min(abs(g - tau) for g in gains) < 1e-9 * max(tau, 1e-300):
            tau *= 1.0 + 1e-6                                   # keep the decision away from ties
        k_star = next((k + 1 for k, g in enumerate(gains) if g < tau), len(gains))
        O, L, n = oracle.attn_early_stop_block(Q, K, V, perm, listed, b, h, i, blk, seg, scale, tau)
        O_ref, L_ref = oracle.attn_block(Q, K, V, perm, listed[:k_star], b, h, i, blk, seg, scale)
        assert n == k_star, (i, tau)
        np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)


@settings(max_examples=20, deadline=None)
@given(seed=st.integers(0, 10_000), tau=st.sampled_from([0.3, 0.6, 0.9, 0.99]))
def test_tau_selection_brute_force_random(seed, tau):
    B, Hq, Hkv, N, d, blk, seg = 1, 1, 1, 96, 8, 8, 24
    Q, K, V = _small(B, Hq, Hkv, N, d, seed=seed, scale=3.0)
    perm = oracle.permute(Q, K, blk, seg)
    counts, lists = oracle.select(Q, K, perm, blk, seg, "tau", tau=tau)
    spb = seg // blk
    scale = 1.0 / (blk * blk * math.sqrt(d))
    for i in range(N // blk):
        s = i // spb
        ncand = s * spb
        if ncand == 0:
            continue
        lc = [_tile_logit_sum(Q, K, perm, 0, 0, i, pb, blk, 1) * scale for pb in range(ncand)]
        ld = [_nat_tile_logit_sum(Q, K, 0, 0, i, j, blk, 1) * scale for j in range(s * spb, i + 1)]
        p = torch.softmax(torch.tensor(lc + ld, dtype=torch.float64), 0).numpy()
        # decisions within 1e-12 of tau are left to rounding on both sides
        cum = np.cumsum(np.sort(p[:ncand])[::-1]) + p[ncand:].sum()
        if np.min(np.abs(cum - tau)) < 1e-12 or abs(p[ncand:].sum() - tau) < 1e-12:
            continue
        assert list(lists[(0, 0, i)]) == _brute_tau(p[ncand:], p[:ncand], set(), tau), i


@settings(max_examples=15, deadline=None)
@given(seed=st.integers(0, 10_000), blk=st.sampled_from([4, 8]), spb=st.sampled_from([2, 3]),
       nseg=st.sampled_from([2, 3]), alpha=st.floats(0.2, 1.0))
def test_select_sample_position_mask_random(seed, blk, spb, nseg, alpha):
    """Random shapes: the block lists are the blocks touched by the
    position-level column/slash mask, restricted to earlier segments."""
    d, seg = 8, blk * spb
    N = seg * nseg
    Q, K, V = _small(1, 1, 1, N, d, seed=seed, scale=2.0)
    counts, lists = oracle.select_sample(Q, K, blk, seg, alpha)
    col, sl = oracle.sample_pattern_scores(Q, K, 0, 0, blk, seg, 1.0 / math.sqrt(d))
    kc, ks = oracle.cumulative_cut(col, alpha), oracle.cumulative_cut(sl, alpha)
    for i in range(N // blk):
        ncand = oracle.n_candidates(i, blk, seg)
        want = {k // blk for q in range(i * blk, (i + 1) * blk) for k in range(ncand * blk)
                if k <= q and (kc[k] or ks[q - k])}
        assert lists[(0, 0, i)].tolist() == sorted(want), i


@settings(max_examples=15, deadline=None)
@given(seed=st.integers(0, 10_000), seg=st.sampled_from([4, 6]), nseg=st.integers(2, 3))
def test_permute_segmented_random(seed, seg, nseg):
    """Random inputs: for query segment s, every key segment before s is in
    descending order of its score against s's summed queries (stable), and
    every later key segment keeps its natural order."""
    d, blk = 8, 2
    N = seg * nseg
    Q, K, V = _small(1, 2, 1, N, d, seed=seed, scale=2.0)
    perm = oracle.permute_segmented(Q, K, blk, seg)
    for t in range(nseg):
        qsum = Q[0, :, t * seg:(t + 1) * seg].astype(np.float64).reshape(-1, d).sum(axis=0)
        sc = K[0, 0].astype(np.float64) @ qsum
        for j in range(nseg):
            got = perm[0, 0, t, j * seg:(j + 1) * seg].tolist()
            if j < t:
                ref = [j * seg + x for x in _brute_force_segment_order(list(sc[j * seg:(j + 1) * seg]))]
            else:
                ref = list(range(j * seg, (j + 1) * seg))
            assert got == ref, (t, j)


@settings(max_examples=12, deadline=None)
@given(seed=st.integers(0, 10_000), keep=st.integers(1, 5), nb=st.integers(2, 8))
def test_gate_brute_force_random(seed, keep, nb):
    """Random inputs: thresholds are the keep-th largest brute-force tile
    maximum (or -inf), and gated attention equals SDPA over the kept tiles
    (the own tile always kept)."""
    blk, d = 4, 8
    N = nb * blk
    Q, K, V = _small(1, 1, 1, N, d, seed=seed, scale=2.0)
    perm = np.arange(N, dtype=np.int32)[None, None].copy()
    _, lists = oracle.dense_lists(1, 1, nb, blk, blk)
    thr = oracle.calibrate_thresholds(Q, K, blk, keep)
    Og, _ = oracle.attn(Q, K, V, perm, lists, blk, blk, gate_thr=thr)
    mask = np.zeros((N, N), bool)
    for i in range(nb):
        qpos = np.arange(i * blk, (i + 1) * blk)
        M = [_brute_tile_max(Q[0, 0, qpos], K[0, 0, j * blk:(j + 1) * blk], qpos, np.arange(j * blk, (j + 1) * blk))
             for j in range(i + 1)]
        t = -math.inf if i + 1 <= keep else sorted(M, reverse=True)[keep - 1]
        assert t == thr[0, 0, i]
        for j in range(i + 1):
            if j == i or M[j] >= t:
                for a in qpos:
                    mask[a, j * blk:min((j + 1) * blk, a + 1)] = True
    ref = _sdpa(Q[0, 0], K[0, 0], V[0, 0], mask=mask)
    assert np.max(np.abs(Og[0, 0] - ref)) < 1e-12
