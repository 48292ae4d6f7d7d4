"""Helpers shared by the GPU parity tests: device transfer, the exactness
preconditions of bit-exact index parity, and the output tolerance check."""
from __future__ import annotations

import functools
import math

import numpy as np
import torch

import oracle
from permuted_block_sparse_b200 import synth

# Output tolerance against the fp64 oracle, given identical block lists.
O_MAX_ABS = 2e-2
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3
# Every partial sum of a score is a multiple of 2^-6 on lattice inputs; below
# 2^18 in magnitude fp32 represents all of them, in any summation order.
EXACT_BOUND = 2.0 ** 18
TAU_MARGIN = 1e-9


def dev(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda()


@functools.lru_cache(maxsize=4)
def workload_inputs(name: str):
    w = synth.WORKLOADS[name]
    Q, K, V, info = synth.make_inputs(w)
    return w, Q, K, V


def assert_key_scores_exact(Q, K, blk):
    """Precondition of bit-exact perm: |qhat| . |k| < 2^18 for every key."""
    Hkv = K.shape[1]
    qhat = oracle.proxy_query(Q, Hkv, blk)
    for b in range(K.shape[0]):
        for h in range(Hkv):
            bound = (np.abs(K[b, h]).astype(np.float64) @ np.abs(qhat[b, h])).max()
            assert bound < EXACT_BOUND, f"key scores not exactly representable: {bound}"


def assert_block_scores_exact(Q, K, perm, blk):
    """Precondition of bit-exact lists: |Qbar| . |Kbar| < 2^18 for all pairs."""
    G = Q.shape[1] // K.shape[1]
    qb = np.abs(oracle.query_block_sums(Q, blk))
    kp = np.abs(oracle.permuted_key_block_sums(K, perm, blk))
    kn = np.abs(oracle.natural_key_block_sums(K, blk))
    for b in range(Q.shape[0]):
        for h in range(Q.shape[1]):
            m1 = (qb[b, h] @ kp[b, h // G].T).max()
            m2 = (qb[b, h] @ kn[b, h // G].T).max()
            assert max(m1, m2) < EXACT_BOUND, f"block scores not exact: {max(m1, m2)}"


def assert_tau_margins(trace: dict, tau: float):
    worst = math.inf
    for (before, after) in trace.values():
        worst = min(worst, abs(after - tau), abs(before - tau))
    assert worst >= TAU_MARGIN, f"a stopping decision is within {worst} of tau"


def pack_lists(counts: np.ndarray, lists: dict, cap: int):
    idx = oracle.lists_to_array(counts, lists, max(cap, 1))
    return torch.from_numpy(counts).cuda(), torch.from_numpy(idx).cuda()


def assert_close(O_gpu: torch.Tensor, O_ref: np.ndarray, rows=None, what=""):
    """max-abs and relative-L2 check over the rows that were computed."""
    g = O_gpu.float().cpu().numpy().astype(np.float64)
    r = O_ref
    if rows is not None:
        g = g[rows]
        r = r[rows]
    ok = ~np.isnan(r)
    g, r = g[ok], r[ok]
    assert g.size > 0
    err = np.abs(g - r)
    max_abs = err.max()
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    assert max_abs <= O_MAX_ABS and rel <= O_REL_L2, f"{what}: max-abs {max_abs:.3e}, rel-L2 {rel:.3e}"
    return max_abs, rel


def block_rows(blocks, blk):
    """Boolean selector helper: list of (b, h, i) -> index arrays for [B,H,N,...]."""
    bs, hs, ns = [], [], []
    for (b, h, i) in blocks:
        for r in range(i * blk, (i + 1) * blk):
            bs.append(b)
            hs.append(h)
            ns.append(r)
    return (np.array(bs), np.array(hs), np.array(ns))


def sample_blocks(w, heads, n_random=6, seed=0):
    """Query blocks checked at full size: first and last, both sides of every
    segment boundary for a few segments, and some random ones."""
    rng = np.random.default_rng(seed)
    nb = w.nb
    spb = w.seg // w.blk
    picks = {0, nb - 1, spb - 1, spb, nb // 2}
    for t in (1, 2, nb // spb - 1):
        picks.add(min(nb - 1, t * spb))
        picks.add(min(nb - 1, t * spb - 1))
    picks |= set(int(x) for x in rng.choice(nb, size=n_random, replace=False))
    return [(b, h, i) for b in range(w.B) for h in heads for i in sorted(picks)]
