#!/usr/bin/env python3
"""Benchmark: permuted block-sparse attention prefill on B200.

One step = pbs_permute + pbs_select + pbs_attn_fwd over one batch of the
128K-token GQA workload (B=1, Hq=32, Hkv=8, d=128, blk 128, seg 4096, 10 %
top-k density, 128 sink keys; planted-stripe lattice inputs), inputs
resident in HBM.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pbs|reference]

Under torchrun each rank runs its own copy of the workload on its own GPU
(weak scaling: the path shards by independent problems, no collective on
the data path); times are the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill attention ms & effective TFLOP/s (% bf16 TC peak) at 128K vs dense"
DEFAULT_WORKLOAD = "llama8b_128k_sink"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="pbs", choices=["pbs", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-dense", action="store_true", help="skip the dense same-kernel comparison run")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="run the workload's settings at this sequence length instead of its own "
                         "(scaled-down cases for counter captures; not a bench line)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def dense_causal_flops(w) -> float:
    return 2.0 * w.d * w.N * w.N * w.Hq * w.B


def selection_label(w) -> str:
    if w.mode == "sample":
        return (f"SampleAttention-style: trunks = last block of each segment, CIA target alpha={w.tau} "
                f"on key columns and slashes, natural key order")
    if w.mode == "gate":
        return f"all earlier blocks, block-max gate calibrated to keep {w.gate_keep} tiles"
    if w.stop_tau > 0:
        return (f"topk density={w.density} in descending block score, early stop at gain < {w.stop_tau}"
                + (", one key permutation per query segment" if w.perm_per_segment else ""))
    sel = f"topk density={w.density}" if w.mode == "topk" else f"tau={w.tau}"
    return (sel + (f" band={w.band}" if w.band else "") + (f" n_sink={w.n_sink}" if w.n_sink else "")
            + (", queries permuted per segment by the guide vector (S2O)" if w.query_perm else ""))


def arm_config(w) -> dict:
    """The workload description both arms print."""
    q_gb = w.B * w.Hq * w.N * w.d * 2 / 1e9
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "blk": w.blk,
            "seg": w.seg, "selection": selection_label(w), "per_gpu": "one full workload per GPU",
            "l2": "inputs larger than L2 (Q alone is %.2f GB)" % q_gb if q_gb > 0.126 else
                  "inputs smaller than L2 (Q is %.3f GB)" % q_gb}


def tile_flops(w) -> float:
    return 4.0 * w.blk * w.blk * w.d


def permute_bytes(w):
    """Algorithmic bytes of pbs_permute: K once, the last query block of every
    head, the permutation written (one per query segment when segmented)."""
    if w.mode in ("gate", "sample"):
        return None
    nseg = (w.N + w.seg - 1) // w.seg
    n_perm = w.B * w.Hkv * w.N * (nseg if w.perm_per_segment else 1)
    q_read = w.B * w.Hq * (w.N if w.perm_per_segment else w.blk) * w.d * 2
    k_read = w.B * w.Hkv * w.N * w.d * 2
    if w.query_perm:
        # the query permutation reads K again (guide vectors) and Q once, and
        # writes qperm
        return 2 * k_read + q_read + w.B * w.Hq * w.N * w.d * 2 + n_perm * 4 + w.B * w.Hq * w.N * 4
    return k_read + q_read + n_perm * 4


def select_bytes(w, cap):
    """Algorithmic bytes of pbs_select (top-k / tau): Q and K once, the pooled
    fp32 block sums written and read back, and the block lists."""
    if w.mode in ("gate", "sample"):
        return None
    pooled = w.B * w.Hq * w.nb * w.d * 4 + 2 * w.B * w.Hkv * w.nb * w.d * 4
    lists = w.B * w.Hq * w.nb * (1 + cap) * 4
    return w.B * w.Hq * w.N * w.d * 2 + w.B * w.Hkv * w.N * w.d * 2 + 2 * pooled + lists


def step_launches(w) -> int:
    """Kernels one step of the workload launches (all in this library)."""
    if w.mode == "gate":
        return 1                                 # attention alone
    if w.mode == "sample":
        return 4                                 # 3 selection kernels + attention
    if w.query_perm:
        return 10                                # 2 + 3 permutation (keys, queries) + 4 selection + attention
    # 2 permutation kernels; selection: query pooling, key pooling (one
    # launch per key permutation), block scores, top-k / cumulative-mass
    # selection; attention
    nperm = (w.N + w.seg - 1) // w.seg if w.perm_per_segment else 1
    return 2 + 3 + nperm + 1


def _gbs(nbytes, ms):
    return None if nbytes is None or ms <= 0 else nbytes / (ms * 1e-3) / 1e9


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML (read-only) while running."""

    REASONS = {
        0x0000000000000001: "gpu_idle", 0x0000000000000002: "applications_clocks_setting",
        0x0000000000000004: "sw_power_cap", 0x0000000000000008: "hw_slowdown",
        0x0000000000000010: "sync_boost", 0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown", 0x0000000000000080: "hw_power_brake_slowdown",
        0x0000000000000100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period: float = 0.02):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self.period = period
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------ CPU baseline
def oracle_baseline(w, Q, K, V, budget_s: float = 20.0, n_blocks: int = 48):
    """Time the fp64 oracle on a bounded sample of the workload.

    Sample: the permutation of one KV head, and the selection and attention
    of ``n_blocks`` query blocks of query head 0 spread evenly over the
    sequence (attention stops early once ``budget_s`` is spent).  A workload
    with at most ``n_blocks`` query blocks in all is run in full.  Scaling
    rule: each part's time is divided by the fraction of that part's work
    the sample covered (1 / (B*Hkv) of the permutation, the sampled share of
    query blocks for selection and attention) and the parts are added; the
    throughput is the dense-causal-equivalent FLOPs over that estimate.
    Returns the seconds actually spent (``sample_s``) beside the estimate."""
    import oracle
    n_rows = w.B * w.Hq * w.nb
    full = n_rows <= n_blocks
    if full:
        blocks = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.nb)]
    else:
        blocks = [(0, 0, int(i)) for i in np.linspace(0, w.nb - 1, n_blocks).round().astype(int)]
    perm_heads = w.B * w.Hkv if full else 1
    f_perm = perm_heads / (w.B * w.Hkv)
    f_sel = len(blocks) / n_rows
    thr = None
    if w.mode == "gate":
        # no permutation or selection step: identity order, every earlier
        # block listed, offline-calibrated thresholds
        t_perm = t_sel = 0.0
        f_perm = f_sel = 1.0
        perm = np.broadcast_to(np.arange(w.N, dtype=np.int32), (w.B, w.Hkv, w.N)).copy()
        lists = {key: np.arange(key[2], dtype=np.int32) for key in blocks}
        thr = np.load(os.path.join(ROOT, "tests", "golden", f"gate_thr_{w.name}.npy")).astype(np.float64)
    elif w.mode == "sample":
        # no permutation: identity order; the selector of one query head
        # (its trunk scores dominate the cost)
        t_perm = 0.0
        f_perm = 1.0
        perm = np.broadcast_to(np.arange(w.N, dtype=np.int32), (w.B, w.Hkv, w.N)).copy()
        t0 = time.perf_counter()
        sel_rows = blocks if full else [(0, 0, i) for i in range(w.nb)]
        _, lists = oracle.select_sample(Q, K, w.blk, w.seg, w.tau, rows=sel_rows)
        t_sel = time.perf_counter() - t0
        f_sel = len(sel_rows) / n_rows
    else:
        t0 = time.perf_counter()
        kv = slice(None) if full else slice(0, 1)
        qh = slice(None) if full else slice(0, w.G)
        if w.perm_per_segment:
            perm1 = oracle.permute_segmented(Q[:, qh], K[:, kv], w.blk, w.seg, w.n_sink)
            perm = np.zeros((w.B, w.Hkv) + perm1.shape[2:], np.int32)
        else:
            perm1 = oracle.permute(Q[:, qh], K[:, kv], w.blk, w.seg, w.n_sink)
            perm = np.zeros((w.B, w.Hkv, w.N), np.int32)
        qsel = Q
        if w.query_perm:
            # the query permutation of the sampled heads (all heads of KV head
            # 0, or all) is part of the permutation step
            qp1 = oracle.permute_queries(Q[:, qh], K[:, kv], w.seg)
            qperm = np.broadcast_to(np.arange(w.N, dtype=np.int32), (w.B, w.Hq, w.N)).copy()
            qperm[:, :qp1.shape[1]] = qp1
            qsel = oracle.gather_queries(Q, qperm)
        t_perm = time.perf_counter() - t0
        perm[:, :perm1.shape[1]] = perm1
        t0 = time.perf_counter()
        counts, lists = oracle.select(qsel, K, perm, w.blk, w.seg, w.mode, density=w.density, tau=w.tau,
                                      band=w.band, n_sink=w.n_sink, rows=blocks,
                                      list_order="score" if w.stop_tau > 0 else "ascending")
        t_sel = time.perf_counter() - t0
    t0 = time.perf_counter()
    done = []
    for key in blocks:
        if w.stop_tau > 0:
            oracle.attn_early_stop(Q, K, V, perm, lists, w.blk, w.seg, w.stop_tau, [key])
        elif w.query_perm:
            b_, h_, i_ = key
            oracle.attn_block_qperm(Q, K, V, perm, qperm, lists.get(key, np.zeros(0, np.int32)), b_, h_, i_,
                                    w.blk, w.seg, 1.0 / math.sqrt(w.d))
        else:
            oracle.attn_blocks(Q, K, V, perm, lists, w.blk, w.seg, [key], gate_thr=thr)
        done.append(key)
        if time.perf_counter() - t0 > budget_s:
            break
    t_attn = time.perf_counter() - t0
    f_attn = len(done) / n_rows
    sample_s = t_perm + t_sel + t_attn
    total = t_perm / f_perm + t_sel / f_sel + t_attn / f_attn
    try:
        from threadpoolctl import threadpool_info
        cores = max([int(x.get("num_threads", 1)) for x in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    if full and len(done) == n_rows:
        what = "the whole workload"
    else:
        parts = []
        if w.mode not in ("gate", "sample"):
            parts.append(f"permutation of {perm_heads} of {w.B * w.Hkv} KV heads")
        if w.mode != "gate":
            parts.append(f"selection of {int(round(f_sel * n_rows))} of {n_rows} query blocks")
        parts.append(f"attention of {len(done)} of {n_rows} query blocks (head 0, spread evenly over N={w.N})")
        what = ", ".join(parts) + "; each part's time divided by its sampled fraction"
    return {
        "value": dense_causal_flops(w) / total / 1e12,
        "unit": "TFLOP/s",
        "cores": cores,
        "kind": "oracle",
        "sample": f"fp64 numpy oracle: {what}; {sample_s:.1f} s timed, est. full run {total:.0f} s",
        "sample_s": sample_s,
        "fraction_of_attention": f_attn,
        "est_full_run_s": total,
    }


# ------------------------------------------------------------------- GPU arm
def run_pbs(args):
    import torch
    import torch.distributed as dist

    import permuted_block_sparse_b200 as pbs
    from permuted_block_sparse_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    pbs.load()

    from permuted_block_sparse_b200 import shard
    w = synth.WORKLOADS[args.workload]
    if args.seq_len:
        if w.mode == "gate" or args.seq_len % w.blk:
            raise SystemExit("--seq-len: a multiple of the block size, and not for the gate workloads "
                             "(their thresholds are calibrated at the workload's own length)")
        w = w.with_(N=args.seq_len)
    Qn, Kn, Vn, _ = synth.make_inputs(w, seed=shard.seed_for_rank(w.seed, rank))
    Q = torch.from_numpy(Qn).to(torch.bfloat16).to(dev)
    K = torch.from_numpy(Kn).to(torch.bfloat16).to(dev)
    V = torch.from_numpy(Vn).to(torch.bfloat16).to(dev)
    s = torch.cuda.current_stream()
    dt = w.tau if w.mode in ("tau", "sample") else w.density
    # the gate workloads list every earlier block (no selection step)
    cap = (max(w.nb - 1, 1) if w.mode == "gate" else
           max(1, pbs.select_capacity(w.N, w.blk, w.seg, w.mode, dt, w.band, w.n_sink)))
    segperm = w.perm_per_segment       # one key permutation per query segment
    nseg = (w.N + w.seg - 1) // w.seg
    perm = torch.empty((w.B, w.Hkv, nseg, w.N) if segperm else (w.B, w.Hkv, w.N), dtype=torch.int32, device=dev)
    counts = torch.empty((w.B, w.Hq, w.nb), dtype=torch.int32, device=dev)
    idx = torch.empty((w.B, w.Hq, w.nb, cap), dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    op_p = pbs.PBS_OP_PERMUTE_SEGMENTED if segperm else pbs.PBS_OP_PERMUTE
    sample = w.mode == "sample"     # SampleAttention-style selection, natural key order
    op_s = (pbs.PBS_OP_SELECT_SEGMENTED if segperm else
            pbs.PBS_OP_SELECT_SAMPLE if sample else pbs.PBS_OP_SELECT)
    ws_p = torch.empty(pbs.workspace_size(op_p, Q, K, w.blk, w.seg) + 256, dtype=torch.uint8, device=dev)
    ws_s = torch.empty(pbs.workspace_size(op_s, Q, K, w.blk, w.seg) + 256, dtype=torch.uint8, device=dev)
    permute = pbs.pbs_permute_segmented if segperm else pbs.pbs_permute
    stats = torch.zeros(2, dtype=torch.int64, device=dev)
    launches_per_step = step_launches(w)
    qperm_on = w.query_perm        # S2O's query permutation
    qperm = ws_q = None
    if qperm_on:
        qperm = torch.empty((w.B, w.Hq, w.N), dtype=torch.int32, device=dev)
        ws_q = torch.empty(pbs.workspace_size(pbs.PBS_OP_PERMUTE_QUERIES, Q, K, w.blk, w.seg) + 256,
                           dtype=torch.uint8, device=dev)
    # Block-max gating workloads: no permutation or selection step; every
    # earlier block is listed and the thresholds (calibrated offline by the
    # oracle, stored beside the tests) decide per tile.
    gate = w.mode == "gate"
    early = w.stop_tau > 0          # S2O early stopping: lists in visiting order
    thr = None
    if gate:
        thr_path = os.path.join(ROOT, "tests", "golden", f"gate_thr_{w.name}.npy")
        thr = torch.from_numpy(np.load(thr_path).astype(np.float32)).to(dev)
        perm.copy_(torch.arange(w.N, dtype=torch.int32, device=dev).expand(w.B, w.Hkv, w.N))
        counts.copy_(torch.arange(w.nb, dtype=torch.int32, device=dev).expand(w.B, w.Hq, w.nb))
        cap = max(w.nb - 1, 1)
        idx = torch.arange(cap, dtype=torch.int32, device=dev).expand(w.B, w.Hq, w.nb, cap).contiguous()
    if sample:
        perm.copy_(torch.arange(w.N, dtype=torch.int32, device=dev).expand(w.B, w.Hkv, w.N))

    ev = {k: [] for k in ("p0", "p1", "s1", "a1")}

    def step(record=False, st=None):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if record else None
        if record and gate:
            e[1] = e[2] = e[0]      # no permutation or selection phase: no events between
        if record:
            e[0].record(s)
        if not gate and not sample:
            permute(Q, K, w.blk, w.seg, w.n_sink, perm=perm, ws=ws_p)
        if qperm_on:
            pbs.pbs_permute_queries(Q, K, w.blk, w.seg, qperm=qperm, ws=ws_q)
        if record and not gate:
            e[1].record(s)
        if qperm_on:
            pbs.pbs_select_qperm(Q, K, perm, qperm, w.blk, w.seg, w.mode, dt, w.n_sink, cap=cap, counts=counts,
                                 idx=idx, ws=ws_s)
        elif not gate:
            pbs.pbs_select(Q, K, None if sample else perm, w.blk, w.seg, w.mode, dt, w.band, w.n_sink, cap=cap,
                           counts=counts, idx=idx, ws=ws_s, score_order=early)
        if record and not gate:
            e[2].record(s)
        if early:
            pbs.pbs_attn_fwd_early_stop(Q, K, V, perm, counts, idx, w.blk, w.seg, w.stop_tau, out=O, lse=lse,
                                        stats=st)
        elif qperm_on:
            pbs.pbs_attn_fwd_qperm(Q, K, V, perm, qperm, counts, idx, w.blk, w.seg, out=O, lse=lse, stats=st)
        else:
            pbs.pbs_attn_fwd(Q, K, V, perm, counts, idx, w.blk, w.seg, out=O, lse=lse, stats=st, gate_thr=thr)
        if record:
            e[3].record(s)
            for k, x in zip(("p0", "p1", "s1", "a1"), e):
                ev[k].append(x)

    # executed tiles (one counted run, outside the timed region)
    step(st=stats)
    pbs.pbs_check_device()
    n_qk, n_gated = int(stats[0]), int(stats[1])
    # gated tiles ran QK^T only; tiles left out by early stopping ran nothing
    n_half = 0 if early else n_gated
    executed_flops = (n_qk - n_half) * tile_flops(w) + n_half * tile_flops(w) / 2
    causal_tiles = w.B * w.Hq * w.nb * (w.nb + 1) // 2

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        t_start.record(s)
        for _ in range(args.steps):
            step(record=True)
        t_end.record(s)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    pbs.pbs_check_device()
    ms_total = t_start.elapsed_time(t_end)
    ms_step = ms_total / args.steps
    ms_perm = statistics.mean(a.elapsed_time(b) for a, b in zip(ev["p0"], ev["p1"]))
    ms_sel = statistics.mean(a.elapsed_time(b) for a, b in zip(ev["p1"], ev["s1"]))
    ms_attn = statistics.mean(a.elapsed_time(b) for a, b in zip(ev["s1"], ev["a1"]))
    if world > 1:
        ms_step, ms_attn = shard.max_over_ranks([ms_step, ms_attn], dist)

    value = dense_causal_flops(w) * world / (ms_step * 1e-3) / 1e12

    # dense causal run of the same kernel: identity permutation, seg = blk,
    # every earlier block listed
    dense = None
    if not args.no_dense and rank == 0:
        ident = torch.arange(w.N, dtype=torch.int32, device=dev).expand(w.B, w.Hkv, w.N).contiguous()
        nb = w.nb
        d_counts = torch.arange(nb, dtype=torch.int32, device=dev).expand(w.B, w.Hq, nb).contiguous()
        d_idx = torch.arange(max(nb - 1, 1), dtype=torch.int32, device=dev).expand(w.B, w.Hq, nb, max(nb - 1, 1)).contiguous()
        Od = torch.empty_like(Q)
        for _ in range(2):
            pbs.pbs_attn_fwd(Q, K, V, ident, d_counts, d_idx, w.blk, w.blk, out=Od, want_lse=False)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        reps = 3
        a.record(s)
        for _ in range(reps):
            pbs.pbs_attn_fwd(Q, K, V, ident, d_counts, d_idx, w.blk, w.blk, out=Od, want_lse=False)
        b.record(s)
        torch.cuda.synchronize()
        pbs.pbs_check_device()
        dms = a.elapsed_time(b) / reps
        dense = {"ms": dms, "tflops": causal_tiles * tile_flops(w) / (dms * 1e-3) / 1e12,
                 "speedup_of_sparse_step": dms / ms_step, "speedup_of_sparse_attention": dms / ms_attn}
        # Attention coverage (outside the timed region): the share of each
        # row's full causal softmax mass on its key set is exp(LSE over the
        # key set - LSE over all causal keys).  The permuted selection of the
        # timed step is compared with the same selection rule on the natural
        # key order (identity permutation) at the same settings.
        if not gate:
            lse_all = torch.empty_like(lse)
            pbs.pbs_attn_fwd(Q, K, V, ident, d_counts, d_idx, w.blk, w.blk, out=Od, lse=lse_all)
            cov_perm = torch.exp(lse - lse_all).flatten()
            q = torch.tensor([0.01, 0.5], device=dev)
            pick = torch.randperm(cov_perm.numel(), device=dev)[:1 << 20]
            pq = torch.quantile(cov_perm[pick], q).tolist()
            if sample:
                # the sample selector already works on the natural key order
                dense["coverage"] = {"selected": {"mean": cov_perm.mean().item(), "p01": pq[0],
                                                  "median": pq[1]},
                                     "what": "share of each query row's causal softmax mass on its key set"}
            else:
                c_nat = torch.empty_like(counts)
                i_nat = torch.empty_like(idx)
                pbs.pbs_select(Q, K, ident, w.blk, w.seg, w.mode, dt, w.band, w.n_sink, cap=cap, counts=c_nat,
                               idx=i_nat, ws=ws_s, score_order=early)
                lse_nat = torch.empty_like(lse)
                if early:
                    pbs.pbs_attn_fwd_early_stop(Q, K, V, ident, c_nat, i_nat, w.blk, w.seg, w.stop_tau, out=Od,
                                                lse=lse_nat)
                else:
                    pbs.pbs_attn_fwd(Q, K, V, ident, c_nat, i_nat, w.blk, w.seg, out=Od, lse=lse_nat)
                pbs.pbs_check_device()
                cov_nat = torch.exp(lse_nat - lse_all).flatten()
                nq = torch.quantile(cov_nat[pick], q).tolist()
                dense["coverage"] = {"permuted": {"mean": cov_perm.mean().item(), "p01": pq[0], "median": pq[1]},
                                     "natural": {"mean": cov_nat.mean().item(), "p01": nq[0], "median": nq[1]},
                                     "what": "share of each query row's causal softmax mass on its key set, "
                                             "permuted keys vs the same rule on natural key order"}
                del c_nat, i_nat, lse_nat
            del lse_all
        del d_idx, Od

    # end to end through the public API with host buffers: H2D of Q, K, V
    # from pinned memory and D2H of O inside the timed region.  HostPrefill
    # overlaps the copies of one KV head's unit with the kernels of another
    # on three streams; the result must equal the device-resident run's O.
    e2e = None
    if not args.no_e2e and qperm_on:
        e2e = {"value": None, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0,
               "note": "the host-memory prefill driver does not take a query permutation"}
    elif not args.no_e2e:
        from permuted_block_sparse_b200.host_pipeline import HostPrefill
        Qh = torch.from_numpy(Qn).to(torch.bfloat16).pin_memory()
        Kh = torch.from_numpy(Kn).to(torch.bfloat16).pin_memory()
        Vh = torch.from_numpy(Vn).to(torch.bfloat16).pin_memory()
        Oh = torch.empty(Qh.shape, dtype=torch.bfloat16).pin_memory()
        hp = HostPrefill(w.B, w.Hq, w.Hkv, w.N, w.d, w.blk, w.seg, "gate" if gate else w.mode, dt, w.band,
                         w.n_sink, w.stop_tau, w.perm_per_segment, gate_thr=thr, device=dev)
        hp.run(Qh, Kh, Vh, Oh)
        torch.cuda.synchronize()
        same = bool(torch.equal(Oh, O.cpu()))
        if world > 1:
            dist.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        k_e2e = max(1, min(args.steps, 5))
        a.record(s)
        for _ in range(k_e2e):
            hp.run(Qh, Kh, Vh, Oh)
        b.record(s)
        torch.cuda.synchronize()
        pbs.pbs_check_device()
        ems = a.elapsed_time(b) / k_e2e
        if world > 1:
            ems = shard.max_over_ranks([ems], dist)[0]
        e2e = {"value": dense_causal_flops(w) * world / (ems * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": ems,
               "h2d_bytes_per_step": int(Qh.numel() * 2 + Kh.numel() * 2 + Vh.numel() * 2),
               "d2h_bytes_per_step": int(Oh.numel() * 2),
               "pipeline": f"{len(hp.units)} units of one KV head, copies and kernels on three streams",
               "matches_device_run": same}
        del hp

    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = executed_flops / (ms_attn * 1e-3) / 1e12
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")
    try:
        with open(os.path.join(ROOT, "permuted_block_sparse_b200", "csrc", "attn_fwd.cu"), "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()[:16]
        with open(tpath) as f:
            tj = json.load(f)
        if tj.get("attn_fwd_sha") == h and tj.get("workload") == w.name:
            traffic = tj.get("bytes_per_launch")
    except Exception:
        traffic = None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = oracle_baseline(w, Qn, Kn, Vn)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": arm_config(w),
        "breakdown": {"permute_ms": ms_perm, "select_ms": ms_sel, "attn_ms": ms_attn,
                      "permute_gbs": _gbs(permute_bytes(w), ms_perm), "select_gbs": _gbs(select_bytes(w, cap), ms_sel),
                      "executed_tiles": n_qk, ("skipped_tiles" if early else "gated_tiles"): n_gated,
                      "causal_tiles": causal_tiles,
                      "density": n_qk / causal_tiles, "executed_tflops": achieved,
                      "effective_tflops": value / world},
        "dense_same_kernel": dense,
        "roofline": {"bound": "tensor", "kernel": "attn_fwd", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"bf16_tflops (burst) of {peak_src}"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clk.summary(),
        "gpu_launches": launches_per_step * args.steps,
    }
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------ reference arm
def run_reference(args):
    """The oracle, as it stands, on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from permuted_block_sparse_b200 import synth
    w = synth.WORKLOADS[args.workload]
    Qn, Kn, Vn, _ = synth.make_inputs(w)
    # each step is one bounded sample of the workload (about per_step s of
    # attention), so the whole run ends within a few minutes
    per_step = max(2.0, 60.0 / max(args.steps + args.warmup, 1))
    # a workload of at most 64 query blocks runs in full; larger ones sample 8
    n_blocks = 64 if w.B * w.Hq * w.nb <= 64 else 8
    for _ in range(args.warmup):
        oracle_baseline(w, Qn, Kn, Vn, budget_s=per_step, n_blocks=n_blocks)
    vals, spent, totals = [], [], []
    cpu = None
    for _ in range(args.steps):
        cpu = oracle_baseline(w, Qn, Kn, Vn, budget_s=per_step, n_blocks=n_blocks)
        vals.append(cpu["value"])
        spent.append(cpu["sample_s"])
        totals.append(cpu["est_full_run_s"])
    value = statistics.median(vals)
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        # the time each step actually ran (its sample), not the full-workload estimate
        "ms_per_step": statistics.median(spent) * 1e3, "est_full_run_s": statistics.median(totals),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu["cores"], "kind": "oracle",
                         "sample": cpu["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_pbs(args)


if __name__ == "__main__":
    main()
