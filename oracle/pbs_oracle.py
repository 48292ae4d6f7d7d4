"""fp64 CPU oracle for permuted block-sparse attention prefill.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package smoke check and
the benchmark's CPU-baseline leg may import this module.  The product path
(the CUDA library and its Python binding) never imports, calls or links it,
and this module imports nothing from the product.

It restates, step by step and in the pages' order, what the method computes:

  1. proxy query + key scores   -- "Sparser Block-Sparse Attention via Token
     Permutation", Technical Summary, 3. Global-Importance-Based Key
     Permutation (Proxy Scoring: the last block of queries, mean-pooled
     attention scores);
  2. segmented stable sort      -- same page, 2. Segmented Permutation for
     Causality and 3. (Sorting: descending within each segment);
  3. block scores               -- same page, 4. Implementation (Block
     Selection by mean pooling on the permuted keys);
  4. top-k / cumulative-mass selection -- same page 4., and "SampleAttention"
     (MLSys 2025 talk), Technical Deep Dive (the attention mass to preserve
     per query);
  5. masked softmax attention   -- "S2O: Early Stopping for Sparse Attention
     via Online Permutation", Technical Summary, 3. Kernel Implementation
     (Pass 1: dense causal window of the current segment; Pass 2: prefix
     keys in permuted order), and the permutation invariance of attention
     (PBS page, 1. Theoretical Foundation);
  6. in-tile block-max gating   -- "Block Sparse Flash Attention", Approach
     (exact QK^T in the tile; skip V and PV when the tile max is below a
     calibrated threshold that keeps roughly the top-k blocks).

Everything is fp64 on the same (bf16-exact) input values.  Where the pages
leave a step open the plainest reading is taken; the readings are:

  * proxy scores are pre-softmax logits of the pooled (summed) proxy query,
    unscaled: the sort is invariant to the positive scale and divisor;
  * the proxy query pools the last ``blk`` query rows of every query head of
    the KV head's group, since keys (and hence the permutation) are per KV
    head;
  * sort ties keep ascending original position (stable);
  * sink positions get score +inf, so they lead segment 0;
  * a query block's own segment is attended densely, in natural order,
    causally (Pass 1); listed permuted blocks come only from earlier
    segments (Pass 2);
  * block score = (sum of the block's query rows) . (sum of the permuted key
    block's rows); for cumulative mass the softmax runs over these scores
    divided by blk^2 * sqrt(d) (the mean tile logit);
  * top-k budget k_i = max(D_i + |F_i|, ceil(rho * n_i)) with rho taken in
    per-mille and the ceiling in integers; ties go to the lower block id;
  * a gated tile is excluded entirely; the query block's own tile is never
    gated; thresholds and tile maxima are raw (unscaled) q.k values.

The variants beside the main path (S2O early stopping, one key permutation
per query segment, S2O's query permutation, the SampleAttention-style
selector, attention coverage) carry their own readings in their docstrings.

Parity pins: tests/test_oracle_pins.py checks every function here against
brute force, closed forms, library routines and invariants.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

F64 = np.float64


# --------------------------------------------------------------------------
# geometry helpers (plain integer bookkeeping)
# --------------------------------------------------------------------------

def segment_of_block(i: int, blk: int, seg: int) -> int:
    """Segment index s(i) of query block i (segments hold seg/blk blocks)."""
    return (i * blk) // seg


def diagonal_blocks(i: int, blk: int, seg: int) -> range:
    """Natural key blocks of block i's own segment that are causal for it."""
    spb = seg // blk
    s = segment_of_block(i, blk, seg)
    return range(s * spb, i + 1)


def n_candidates(i: int, blk: int, seg: int) -> int:
    """Number of permuted key blocks in segments strictly before s(i)."""
    spb = seg // blk
    return segment_of_block(i, blk, seg) * spb


def topk_target(n_causal: int, density: float) -> int:
    """ceil(rho * n) with rho rounded to per-mille, computed in integers."""
    r = int(round(1000.0 * density))
    return -((-r * n_causal) // 1000)


# --------------------------------------------------------------------------
# 1-2. permutation
# --------------------------------------------------------------------------

def proxy_query(Q: np.ndarray, Hkv: int, blk: int) -> np.ndarray:
    """qhat[b, hkv, :] = sum over the last ``blk`` query rows of every query
    head in KV head hkv's group.  Q: [B, Hq, N, d].  Returns fp64 [B, Hkv, d]."""
    B, Hq, N, d = Q.shape
    G = Hq // Hkv
    out = np.zeros((B, Hkv, d), F64)
    for b in range(B):
        for h in range(Hkv):
            rows = Q[b, h * G:(h + 1) * G, N - blk:N, :].astype(F64)
            out[b, h] = rows.reshape(-1, d).sum(axis=0)
    return out


def key_scores(qhat: np.ndarray, K: np.ndarray, n_sink: int = 0) -> np.ndarray:
    """s[b, hkv, j] = qhat[b, hkv] . K[b, hkv, j] in fp64; sinks get +inf."""
    B, Hkv, N, d = K.shape
    s = np.zeros((B, Hkv, N), F64)
    for b in range(B):
        for h in range(Hkv):
            s[b, h] = K[b, h].astype(F64) @ qhat[b, h]
    if n_sink > 0:
        s[:, :, :n_sink] = np.inf
    return s


def sort_segments(scores: np.ndarray, seg: int) -> np.ndarray:
    """perm[b, h, p] = original position at logical position p.

    Within each segment [t*seg, min((t+1)*seg, N)) positions are ordered by
    descending score, equal scores in ascending position; segment order is
    kept, so perm is a bijection of each segment onto itself."""
    B, H, N = scores.shape
    perm = np.empty((B, H, N), np.int32)
    for b in range(B):
        for h in range(H):
            for lo in range(0, N, seg):
                hi = min(lo + seg, N)
                order = np.argsort(-scores[b, h, lo:hi], kind="stable")
                perm[b, h, lo:hi] = lo + order
    return perm


def permute(Q: np.ndarray, K: np.ndarray, blk: int, seg: int, n_sink: int = 0) -> np.ndarray:
    """The full permutation step: proxy query, key scores, segment sort."""
    Hkv = K.shape[1]
    qhat = proxy_query(Q, Hkv, blk)
    return sort_segments(key_scores(qhat, K, n_sink), seg)


def segment_queries(Q: np.ndarray, Hkv: int, seg: int) -> np.ndarray:
    """qbar[b, hkv, s, :] = sum of every query row of segment s of every
    query head in KV head hkv's group (fp64): the segment's representative
    query.  Returns [B, Hkv, nseg, d]."""
    B, Hq, N, d = Q.shape
    G = Hq // Hkv
    nseg = (N + seg - 1) // seg
    out = np.zeros((B, Hkv, nseg, d), F64)
    for b in range(B):
        for h in range(Hkv):
            for t in range(nseg):
                rows = Q[b, h * G:(h + 1) * G, t * seg:min((t + 1) * seg, N), :].astype(F64)
                out[b, h, t] = rows.reshape(-1, d).sum(axis=0)
    return out


def permute_segmented(Q: np.ndarray, K: np.ndarray, blk: int, seg: int, n_sink: int = 0) -> np.ndarray:
    """One key permutation per query segment (S2O's historical KV permutation).

    "S2O: Early Stopping for Sparse Attention via Online Permutation",
    Technical Summary, 1. Online Permutation via Index-Driven Loading: each
    query segment ranks the keys that precede it by one query standing for
    the whole segment.  For query segment s the keys are scored against that
    query (segment_queries; sinks
    get +inf); each key segment before s is sorted by those scores
    (descending, ties in ascending position); key segments from s on are not
    s's history and keep their natural order.  Returns perm[b, hkv, s, p],
    [B, Hkv, nseg, N] int32."""
    B, Hkv, N, d = K.shape
    qs = segment_queries(Q, Hkv, seg)
    nseg = qs.shape[2]
    out = np.empty((B, Hkv, nseg, N), np.int32)
    for t in range(nseg):
        sc = key_scores(qs[:, :, t], K, n_sink)
        srt = sort_segments(sc, seg)
        out[:, :, t] = np.arange(N, dtype=np.int32)
        out[:, :, t, :t * seg] = srt[:, :, :t * seg]
    return out


def perm_for_block(perm: np.ndarray, b: int, hk: int, i: int, blk: int, seg: int) -> np.ndarray:
    """The key permutation query block i reads: the KV head's ([B, Hkv, N]),
    or its query segment's ([B, Hkv, nseg, N], permute_segmented)."""
    if perm.ndim == 3:
        return perm[b, hk]
    return perm[b, hk, segment_of_block(i, blk, seg)]


# --------------------------------------------------------------------------
# 3-4. block selection
# --------------------------------------------------------------------------

def query_block_sums(Q: np.ndarray, blk: int) -> np.ndarray:
    """Qbar[b, hq, i] = sum of the blk rows of query block i (fp64)."""
    B, H, N, d = Q.shape
    return Q.astype(F64).reshape(B, H, N // blk, blk, d).sum(axis=3)


def permuted_key_block_sums(K: np.ndarray, perm: np.ndarray, blk: int) -> np.ndarray:
    """Kbar[b, hkv, pb] = sum of K rows perm[pb*blk .. pb*blk+blk-1] (fp64)."""
    B, H, N, d = K.shape
    out = np.zeros((B, H, N // blk, d), F64)
    for b in range(B):
        for h in range(H):
            rows = K[b, h].astype(F64)[perm[b, h]]
            out[b, h] = rows.reshape(N // blk, blk, d).sum(axis=1)
    return out


def natural_key_block_sums(K: np.ndarray, blk: int) -> np.ndarray:
    B, H, N, d = K.shape
    return K.astype(F64).reshape(B, H, N // blk, blk, d).sum(axis=3)


def inverse_permutation(perm_row: np.ndarray) -> np.ndarray:
    """inv[perm[p]] = p: the logical position of each original position."""
    inv = np.empty_like(perm_row)
    inv[perm_row] = np.arange(perm_row.shape[0], dtype=perm_row.dtype)
    return inv


def forced_blocks(i: int, inv_row: np.ndarray, blk: int, seg: int,
                  band: int, n_sink: int) -> List[int]:
    """Permuted blocks of earlier segments that must be listed for block i:
    those holding a sink position (< n_sink) or a position among the ``band``
    most recent keys of any query in the block.  ``inv_row`` is the inverse
    of the KV head's permutation.  Ascending block ids."""
    ncand = n_candidates(i, blk, seg)
    if ncand == 0:
        return []
    s_start = segment_of_block(i, blk, seg) * seg
    want = set()
    if n_sink > 0:
        for pos in range(0, min(n_sink, s_start)):
            want.add(int(inv_row[pos]) // blk)
    if band > 0:
        lo = max(0, i * blk - band + 1)
        for pos in range(lo, s_start):
            want.add(int(inv_row[pos]) // blk)
    return sorted(pb for pb in want if pb < ncand)


def select(Q: np.ndarray, K: np.ndarray, perm: np.ndarray, blk: int, seg: int,
           mode: str, density: float = 1.0, tau: float = 1.0, band: int = 0,
           n_sink: int = 0, rows: Optional[Iterable[Tuple[int, int, int]]] = None,
           trace: Optional[dict] = None, list_order: str = "ascending"):
    """Per (b, hq, i) lists of permuted key blocks to attend.

    Returns (counts [B,Hq,nb] int32, lists dict {(b,hq,i): int32 array}).
    With ``rows`` given, only those (b, hq, i) are computed (others count 0).
    mode "topk": budget from ``density``; mode "tau": cumulative mass.
    With ``trace`` (a dict), tau mode records per row the accumulated mass
    before the last added block and after it, so callers can check how far
    each stopping decision is from tau.
    list_order "ascending": lists sorted by block id; "score": the forced
    blocks first (ascending), then the other chosen blocks by descending
    block score, ties to the lower block id -- the visiting order of S2O's
    Pass 2, which processes candidates in descending estimated importance
    ("S2O: Early Stopping for Sparse Attention via Online Permutation",
    Technical Summary, 2. Early-Stopping Rule)."""
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    nb = N // blk
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(nb)]
    rows = list(rows)
    counts = np.zeros((B, Hq, nb), np.int32)
    lists = {}
    kbar_p = {}
    kbar_n = {}
    inv = {}
    qbar_cache = {}
    for (b, h, i) in rows:
        hk = h // G
        pkey = (b, hk) if perm.ndim == 3 else (b, hk, segment_of_block(i, blk, seg))
        if pkey not in kbar_p:
            prow = perm_for_block(perm, b, hk, i, blk, seg)
            kbar_p[pkey] = permuted_key_block_sums(K[b:b + 1, hk:hk + 1], prow[None, None], blk)[0, 0]
            inv[pkey] = inverse_permutation(prow)
        if (b, hk) not in kbar_n:
            kbar_n[(b, hk)] = natural_key_block_sums(K[b:b + 1, hk:hk + 1], blk)[0, 0]
        if (b, h) not in qbar_cache:
            qbar_cache[(b, h)] = query_block_sums(Q[b:b + 1, h:h + 1], blk)[0, 0]
        qb = qbar_cache[(b, h)][i]
        ncand = n_candidates(i, blk, seg)
        diag = list(diagonal_blocks(i, blk, seg))
        D = len(diag)
        if ncand == 0:
            lists[(b, h, i)] = np.zeros(0, np.int32)
            continue
        S = kbar_p[pkey][:ncand] @ qb                         # exact on lattice inputs
        F = forced_blocks(i, inv[pkey], blk, seg, band, n_sink)
        rest = np.setdiff1d(np.arange(ncand, dtype=np.int64), np.array(F, np.int64))
        # descending score, ties to the lower block id
        order = rest[np.lexsort((rest, -S[rest]))] if rest.size else rest
        if mode == "topk":
            k = max(D + len(F), topk_target(i + 1, density))
            take = k - D - len(F)
            chosen = list(F) + [int(x) for x in order[:take]]
        elif mode == "tau":
            if tau >= 1.0:
                chosen = list(range(ncand))
            else:
                scale = 1.0 / (blk * blk * math.sqrt(d))
                lg_c = S * scale
                lg_d = np.array([kbar_n[(b, hk)][j] @ qb for j in diag], F64) * scale
                m = max(lg_c.max(), lg_d.max())
                e_c = np.exp(lg_c - m)
                e_d = np.exp(lg_d - m)
                Z = e_c.sum() + e_d.sum()
                cum = (e_d.sum() + e_c[F].sum()) / Z if F else e_d.sum() / Z
                chosen = list(F)
                before = cum
                for pb in order:
                    if cum >= tau:
                        break
                    chosen.append(int(pb))
                    before = cum
                    cum += e_c[pb] / Z
                if trace is not None:
                    trace[(b, h, i)] = (before, cum)
        else:
            raise ValueError(mode)
        if list_order == "ascending":
            arr = np.array(sorted(chosen), np.int32)
        elif list_order == "score":
            fset = set(int(x) for x in F)
            lead = sorted(x for x in chosen if x in fset)
            tail = sorted((x for x in chosen if x not in fset), key=lambda x: (-S[x], x))
            arr = np.array(lead + tail, np.int32)
        else:
            raise ValueError(list_order)
        lists[(b, h, i)] = arr
        counts[b, h, i] = arr.size
    return counts, lists


def sample_trunk_rows(N: int, blk: int, seg: int) -> np.ndarray:
    """SampleAttention's sampled queries: one trunk per segment, its last
    query block (the rows that see the segment's whole history)."""
    rows = []
    for lo in range(0, N, seg):
        hi = min(lo + seg, N)
        rows.extend(range(hi - blk, hi))
    return np.array(rows, np.int64)


def sample_pattern_scores(Q, K, b: int, hq: int, blk: int, seg: int, scale: float):
    """Stage 1 ("SampleAttention", Technical Deep Dive, 1. Trunk Sampling):
    the softmax probabilities of the sampled rows over every key they see
    (fp64), summed per key column and per slash offset q - k.  Returns
    (col [N], slash [N])."""
    Hq, Hkv = Q.shape[1], K.shape[1]
    hk = hq // (Hq // Hkv)
    N = Q.shape[2]
    col = np.zeros(N, F64)
    sl = np.zeros(N, F64)
    Kf = K[b, hk].astype(F64)
    for q in sample_trunk_rows(N, blk, seg):
        lg = (Kf[:q + 1] @ Q[b, hq, q].astype(F64)) * scale
        e = np.exp(lg - lg.max())
        p = e / e.sum()
        col[:q + 1] += p
        sl[:q + 1] += p[::-1]                    # offset q - k for k = q .. 0
    return col, sl


def cumulative_cut(score: np.ndarray, alpha: float) -> np.ndarray:
    """Stage 2 decoupled filtering for one pattern family: the entries in
    descending score (ties to the lower index) up to and including the one
    at which the accumulated score first reaches alpha of the total; alpha
    >= 1 keeps every entry with a positive score.  Boolean mask."""
    keep = np.zeros(score.size, bool)
    order = np.lexsort((np.arange(score.size), -score))
    total = score.sum()
    if alpha >= 1.0:
        keep[score > 0] = True
        return keep
    acc = 0.0
    for x in order:
        if acc >= alpha * total:
            break
        keep[x] = True
        acc += score[x]
    return keep


def select_sample(Q, K, blk: int, seg: int, alpha: float,
                  rows: Optional[Iterable[Tuple[int, int, int]]] = None, trace: Optional[dict] = None):
    """A SampleAttention-style selector over natural key blocks ("SampleAttention",
    Technical Deep Dive, Stage 1 Trunk Sampling and Stage 2 Score-Based
    Filtering).  Per (b, hq): Stage 1 scores (sample_pattern_scores); kept
    key columns and kept slash offsets by decoupled cumulative cuts at alpha
    of each family's total (the CIA target for both); query block i lists
    every earlier-segment key block that holds a kept column or a key q - d
    of one of its queries q and a kept offset d.  Lists ascending, natural
    key order (attend with the identity permutation).  ``trace`` receives,
    per (b, hq) and family, the accumulated score before and after the last
    kept entry, alpha times the total, and the scores of the last kept and
    the first dropped entry, for margin checks."""
    B, Hq, N, d = Q.shape
    nb = N // blk
    scale = 1.0 / math.sqrt(d)
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(nb)]
    rows = list(rows)
    counts = np.zeros((B, Hq, nb), np.int32)
    lists = {}
    kept = {}
    for (b, h, i) in rows:
        if (b, h) not in kept:
            col, sl = sample_pattern_scores(Q, K, b, h, blk, seg, scale)
            kc, ks = cumulative_cut(col, alpha), cumulative_cut(sl, alpha)
            kept[(b, h)] = (kc, ks)
            if trace is not None:
                tr = []
                for sc, kp in ((col, kc), (sl, ks)):
                    order = np.lexsort((np.arange(sc.size), -sc))
                    n = int(kp.sum())
                    before = sc[order[:n - 1]].sum() if n > 0 else 0.0
                    last = sc[order[n - 1]] if n > 0 else np.inf
                    nxt = sc[order[n]] if n < sc.size else -np.inf
                    tr.append((before, sc[order[:n]].sum(), alpha * sc.sum(), last, nxt))
                trace[(b, h)] = tr
        kc, ks = kept[(b, h)]
        ncand = n_candidates(i, blk, seg)
        chosen = set()
        for j in range(ncand):
            if kc[j * blk:(j + 1) * blk].any():
                chosen.add(j)
        q0 = i * blk
        for dlt in np.nonzero(ks)[0]:
            lo, hi = q0 - int(dlt), q0 + blk - 1 - int(dlt)
            if hi < 0:
                continue
            for j in range(max(lo, 0) // blk, min(hi // blk, ncand - 1) + 1):
                chosen.add(j)
        arr = np.array(sorted(chosen), np.int32)
        lists[(b, h, i)] = arr
        counts[b, h, i] = arr.size
    return counts, lists


def guide_vectors(K: np.ndarray) -> np.ndarray:
    """S2O's shared guide vector for ranking queries ("S2O: Early Stopping
    for Sparse Attention via Online Permutation", Technical Summary, 1.
    Online Permutation via Index-Driven Loading, Query Permutation).  Read
    here as the sum of every key of the KV head, so that a query's score
    q . g is the sum of its logits over all keys: large for the queries that
    attend broadly, which draw horizontal stripes.  fp64 [B, Hkv, d]."""
    return K.astype(F64).sum(axis=2)


def permute_queries(Q: np.ndarray, K: np.ndarray, seg: int) -> np.ndarray:
    """Q_perm: per (b, query head, segment), the query positions in
    descending q . g (g the KV head's guide vector), equal scores in ascending
    position.  qperm[b, hq, p] = original query position at permuted
    position p; a bijection of each segment onto itself.  [B, Hq, N] int32."""
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    g = guide_vectors(K)
    sc = np.zeros((B, Hq, N), F64)
    for b in range(B):
        for h in range(Hq):
            sc[b, h] = Q[b, h].astype(F64) @ g[b, h // G]
    return sort_segments(sc, seg)


def gather_queries(Q: np.ndarray, qperm: np.ndarray) -> np.ndarray:
    """Qp[b, hq, p] = Q[b, hq, qperm[b, hq, p]]: the queries in permuted
    order.  Selection on Qp pools each permuted query block."""
    B, Hq, N, d = Q.shape
    Qp = np.empty_like(Q)
    for b in range(B):
        for h in range(Hq):
            Qp[b, h] = Q[b, h, qperm[b, h]]
    return Qp


def attn_block_qperm(Q, K, V, perm, qperm, listed, b, hq, i, blk, seg, scale):
    """O [blk, d] and LSE [blk] (fp64) for permuted query block i of (b, hq):
    rows are the queries at positions qperm[b, hq, i*blk + r].  Each row q
    attends the keys of its own segment up to q (natural order, causal, as
    in S2O's Pass 1) and the keys of the listed permuted blocks (all in
    earlier segments).  Row r's results belong at position qperm[..]."""
    Hq, Hkv = Q.shape[1], K.shape[1]
    hk = hq // (Hq // Hkv)
    q_pos = qperm[b, hq, i * blk:(i + 1) * blk].astype(np.int64)
    q = Q[b, hq, q_pos].astype(F64)
    s0 = segment_of_block(i, blk, seg) * seg
    perm_row = perm_for_block(perm, b, hk, i, blk, seg)
    keys = [perm_row[pb * blk:(pb + 1) * blk].astype(np.int64) for pb in listed]
    keys.append(np.arange(s0, q_pos.max() + 1, dtype=np.int64))
    keys = np.concatenate(keys)
    vis = keys[None, :] <= q_pos[:, None]
    logits = np.where(vis, (q @ K[b, hk, keys].astype(F64).T) * scale, -np.inf)
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    l = e.sum(axis=1, keepdims=True)
    return (e @ V[b, hk, keys].astype(F64)) / l, (m + np.log(l))[:, 0]


def attn_qperm(Q, K, V, perm, qperm, lists: dict, blk: int, seg: int, scale: Optional[float] = None):
    """O [B,Hq,N,d] and LSE [B,Hq,N] (fp64) at the queries' original
    positions, for lists indexed by permuted query block (b, hq, i)."""
    B, Hq, N, d = Q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.full((B, Hq, N, d), np.nan, F64)
    L = np.full((B, Hq, N), np.nan, F64)
    for b in range(B):
        for h in range(Hq):
            for i in range(N // blk):
                listed = lists.get((b, h, i), np.zeros(0, np.int32))
                o, lse = attn_block_qperm(Q, K, V, perm, qperm, listed, b, h, i, blk, seg, scale)
                pos = qperm[b, h, i * blk:(i + 1) * blk]
                O[b, h, pos] = o
                L[b, h, pos] = lse
    return O, L


def lists_to_array(counts: np.ndarray, lists: dict, cap: int) -> np.ndarray:
    """Pack lists into idx[B,Hq,nb,cap] (unused entries -1)."""
    B, H, nb = counts.shape
    idx = np.full((B, H, nb, cap), -1, np.int32)
    for (b, h, i), arr in lists.items():
        idx[b, h, i, :arr.size] = arr
    return idx


# --------------------------------------------------------------------------
# 5-6. attention (optionally gated)
# --------------------------------------------------------------------------

def key_tiles(i: int, listed: Sequence[int], perm_row: np.ndarray, blk: int, seg: int):
    """The tiles query block i visits: (kind, id, key positions).

    kind "perm": permuted block of an earlier segment, keys perm[pb*blk ...];
    kind "diag": natural block of the block's own segment."""
    tiles = []
    for pb in listed:
        tiles.append(("perm", int(pb), perm_row[pb * blk:(pb + 1) * blk].astype(np.int64)))
    for j in diagonal_blocks(i, blk, seg):
        tiles.append(("diag", j, np.arange(j * blk, (j + 1) * blk, dtype=np.int64)))
    return tiles


def attn_block(Q, K, V, perm, listed, b, hq, i, blk, seg, scale,
               gate_thr: Optional[float] = None):
    """O and LSE (natural log of the softmax normaliser of the scaled logits)
    for the ``blk`` query rows of block i of (b, hq), fp64.

    The key set is the listed permuted blocks plus the causal part of the
    block's own segment; with ``gate_thr`` every tile except block i's own is
    dropped when its maximal raw q.k over visible entries is below it."""
    Hq, Hkv = Q.shape[1], K.shape[1]
    hk = hq // (Hq // Hkv)
    q_pos = np.arange(i * blk, (i + 1) * blk)
    q = Q[b, hq, i * blk:(i + 1) * blk].astype(F64)
    keys, kmask = [], []
    for kind, tid, pos in key_tiles(i, listed, perm_for_block(perm, b, hk, i, blk, seg), blk, seg):
        visible = pos[None, :] <= q_pos[:, None]
        if gate_thr is not None and not (kind == "diag" and tid == i):
            raw = q @ K[b, hk, pos].astype(F64).T
            tmax = raw[visible].max() if visible.any() else -np.inf
            if tmax < gate_thr:
                continue
        keys.append(pos)
        kmask.append(visible)
    keys = np.concatenate(keys)
    vis = np.concatenate(kmask, axis=1)
    logits = (q @ K[b, hk, keys].astype(F64).T) * scale
    logits = np.where(vis, logits, -np.inf)
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    l = e.sum(axis=1, keepdims=True)
    O = (e @ V[b, hk, keys].astype(F64)) / l
    lse = (m + np.log(l))[:, 0]
    return O, lse


def attn(Q, K, V, perm, lists: dict, blk: int, seg: int, scale: Optional[float] = None,
         gate_thr: Optional[np.ndarray] = None, blocks: Optional[Iterable[Tuple[int, int, int]]] = None):
    """O [B,Hq,N,d] and LSE [B,Hq,N] (fp64) over the given (b, hq, i) blocks
    (all by default; rows of other blocks stay NaN).  ``lists`` maps
    (b, hq, i) to its listed permuted blocks (missing = none)."""
    B, Hq, N, d = Q.shape
    nb = N // blk
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if blocks is None:
        blocks = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(nb)]
    O = np.full((B, Hq, N, d), np.nan, F64)
    L = np.full((B, Hq, N), np.nan, F64)
    for (b, h, i) in blocks:
        listed = lists.get((b, h, i), np.zeros(0, np.int32))
        thr = None if gate_thr is None else float(gate_thr[b, h, i])
        o, lse = attn_block(Q, K, V, perm, listed, b, h, i, blk, seg, scale, thr)
        O[b, h, i * blk:(i + 1) * blk] = o
        L[b, h, i * blk:(i + 1) * blk] = lse
    return O, L


def attn_blocks(Q, K, V, perm, lists: dict, blk: int, seg: int, blocks: Iterable[Tuple[int, int, int]],
                scale: Optional[float] = None, gate_thr: Optional[np.ndarray] = None) -> dict:
    """{(b, hq, i): (O [blk, d], LSE [blk])} for the given query blocks only."""
    d = Q.shape[3]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = {}
    for (b, h, i) in blocks:
        listed = lists.get((b, h, i), np.zeros(0, np.int32))
        thr = None if gate_thr is None else float(gate_thr[b, h, i])
        out[(b, h, i)] = attn_block(Q, K, V, perm, listed, b, h, i, blk, seg, scale, thr)
    return out


def attn_early_stop_block(Q, K, V, perm, listed, b, hq, i, blk, seg, scale, stop_tau: float,
                          trace: Optional[list] = None):
    """S2O's two passes with the early-stopping rule, fp64, for the ``blk``
    query rows of block i of (b, hq).  Returns (O, LSE, tiles of Pass 2 run).

    "S2O: Early Stopping for Sparse Attention via Online Permutation",
    Technical Summary, 3. Kernel Implementation and 2. Early-Stopping Rule:
    Pass 1 runs dense causal attention over the block's own segment (natural
    order) and leaves the online-softmax state (m, l, acc) per query row;
    Pass 2 continues from that state over the listed permuted blocks in the
    order given.  After each Pass-2 tile the marginal gain of every row is
    dl / l, the tile's exponential mass over the accumulated mass (both in
    the running-max frame, so the ratio does not depend on the frame); when
    the largest gain over the block's rows is below ``stop_tau`` the
    remaining listed blocks are skipped (the tile just run stays in).
    ``trace``, if given, receives the largest gain of every tile run."""
    Hq, Hkv = Q.shape[1], K.shape[1]
    hk = hq // (Hq // Hkv)
    q_pos = np.arange(i * blk, (i + 1) * blk)
    q = Q[b, hq, i * blk:(i + 1) * blk].astype(F64)
    # Pass 1: natural keys of the own segment up to the block's end, causal
    s0 = segment_of_block(i, blk, seg) * seg
    own = np.arange(s0, (i + 1) * blk, dtype=np.int64)
    lg = (q @ K[b, hk, own].astype(F64).T) * scale
    lg = np.where(own[None, :] <= q_pos[:, None], lg, -np.inf)
    m = lg.max(axis=1)
    e = np.exp(lg - m[:, None])
    l = e.sum(axis=1)
    acc = e @ V[b, hk, own].astype(F64)
    # Pass 2: listed permuted blocks in the given order (all keys visible)
    n_run = 0
    prow = perm_for_block(perm, b, hk, i, blk, seg)
    for pb in listed:
        pos = prow[int(pb) * blk:(int(pb) + 1) * blk].astype(np.int64)
        lg = (q @ K[b, hk, pos].astype(F64).T) * scale
        m_new = np.maximum(m, lg.max(axis=1))
        alpha = np.exp(m - m_new)
        e = np.exp(lg - m_new[:, None])
        dl = e.sum(axis=1)
        l = l * alpha + dl
        acc = acc * alpha[:, None] + e @ V[b, hk, pos].astype(F64)
        m = m_new
        n_run += 1
        gain = float((dl / l).max())
        if trace is not None:
            trace.append(gain)
        if gain < stop_tau:
            break
    return acc / l[:, None], m + np.log(l), n_run


def attn_early_stop(Q, K, V, perm, lists: dict, blk: int, seg: int, stop_tau: float,
                    blocks: Iterable[Tuple[int, int, int]], scale: Optional[float] = None,
                    traces: Optional[dict] = None) -> dict:
    """{(b, hq, i): (O [blk, d], LSE [blk], Pass-2 tiles run)} for the given
    blocks; ``lists`` must hold each block's list in visiting order."""
    d = Q.shape[3]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = {}
    for (b, h, i) in blocks:
        listed = lists.get((b, h, i), np.zeros(0, np.int32))
        tr = [] if traces is not None else None
        out[(b, h, i)] = attn_early_stop_block(Q, K, V, perm, listed, b, h, i, blk, seg, scale, stop_tau, tr)
        if traces is not None:
            traces[(b, h, i)] = tr
    return out


def coverage_block(Q, K, perm, listed, b, hq, i, blk, seg, scale) -> np.ndarray:
    """Per query row of block i: the share of the row's full causal softmax
    mass that falls on the block's key set (the own segment's causal keys
    and the listed permuted blocks), fp64 from explicit exponentials.

    This is the attention-coverage measure behind "Sparser Block-Sparse
    Attention via Token Permutation", Key Results (fewer blocks for the same
    coverage once keys are permuted)."""
    Hq, Hkv = Q.shape[1], K.shape[1]
    hk = hq // (Hq // Hkv)
    q_pos = np.arange(i * blk, (i + 1) * blk)
    q = Q[b, hq, i * blk:(i + 1) * blk].astype(F64)
    keys = np.arange((i + 1) * blk)
    lg = (q @ K[b, hk, keys].astype(F64).T) * scale
    vis = keys[None, :] <= q_pos[:, None]
    lg = np.where(vis, lg, -np.inf)
    m = lg.max(axis=1, keepdims=True)
    e = np.exp(lg - m)
    inset = np.zeros(keys.size, bool)
    for _, _, pos in key_tiles(i, listed, perm_for_block(perm, b, hk, i, blk, seg), blk, seg):
        inset[pos] = True
    return (e * inset[None, :]).sum(axis=1) / e.sum(axis=1)


# --------------------------------------------------------------------------
# 6. gate calibration
# --------------------------------------------------------------------------

def tile_maxima(Q, K, b, hq, i, blk) -> np.ndarray:
    """M[j] = max over visible (q, k) of raw q.k for natural tiles j <= i."""
    Hq, Hkv = Q.shape[1], K.shape[1]
    hk = hq // (Hq // Hkv)
    q = Q[b, hq, i * blk:(i + 1) * blk].astype(F64)
    k = K[b, hk, :(i + 1) * blk].astype(F64)
    raw = q @ k.T
    q_pos = np.arange(i * blk, (i + 1) * blk)[:, None]
    k_pos = np.arange((i + 1) * blk)[None, :]
    raw = np.where(k_pos <= q_pos, raw, -np.inf)
    return raw.reshape(blk, i + 1, blk).max(axis=(0, 2))


def calibrate_thresholds(Q, K, blk: int, keep: int,
                         blocks: Optional[Iterable[Tuple[int, int, int]]] = None) -> np.ndarray:
    """thr[b, hq, i] = the keep-th largest causal tile maximum of block i
    (-inf when block i has at most ``keep`` causal tiles).  Unlisted blocks
    (when ``blocks`` is given) get -inf."""
    B, Hq, N, d = Q.shape
    nb = N // blk
    thr = np.full((B, Hq, nb), -np.inf, F64)
    if blocks is None:
        blocks = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(nb)]
    for (b, h, i) in blocks:
        if i + 1 <= keep:
            continue
        M = tile_maxima(Q, K, b, h, i, blk)
        thr[b, h, i] = np.sort(M)[::-1][keep - 1]
    return thr


def dense_lists(B: int, Hq: int, nb: int, blk: int, seg: int) -> Tuple[np.ndarray, dict]:
    """Every candidate block listed (density 1): dense causal attention."""
    counts = np.zeros((B, Hq, nb), np.int32)
    lists = {}
    for b in range(B):
        for h in range(Hq):
            for i in range(nb):
                arr = np.arange(n_candidates(i, blk, seg), dtype=np.int32)
                lists[(b, h, i)] = arr
                counts[b, h, i] = arr.size
    return counts, lists
