"""Prefill from host memory: pinned Q, K, V in, pinned O out.

The work is split into units of (batch, contiguous range of KV heads with
their query heads).  Units are independent (a KV head's permutation, its
query heads' block lists and their attention read no other unit's data), so
three CUDA streams overlap them: while the GPU computes unit u, the
host-to-device copies of unit u + 1 and the device-to-host copy of unit u - 1
are in flight.  Every step of the path still runs in the library's kernels;
this module only places the copies and launches on streams and orders them
with events.  A unit's results are bit-identical to the same heads of one
whole-tensor call.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _binding as bd


class HostPrefill:
    """Device buffers, streams and events for repeated prefills of one shape.

    ``mode`` is "topk" or "tau" (permute + select + attention), "sample"
    (the SampleAttention-style selector + attention in natural key order) or
    "gate" (seg == blk, every earlier block listed, the block-max gate with
    ``gate_thr``, a float32 device tensor [B, Hq, N / blk]).  ``stop_tau`` > 0 selects S2O
    early stopping (lists in visiting order); ``perm_per_segment`` one key
    permutation per query segment.  ``heads_per_chunk`` KV heads form a unit.
    """

    def __init__(self, B: int, Hq: int, Hkv: int, N: int, d: int, blk: int, seg: int, mode: str = "topk",
                 density_or_tau: float = 1.0, band: int = 0, n_sink: int = 0, stop_tau: float = 0.0,
                 perm_per_segment: bool = False, gate_thr: Optional[torch.Tensor] = None,
                 heads_per_chunk: int = 1, device: Optional[torch.device] = None):
        if mode not in ("topk", "tau", "sample", "gate"):
            raise ValueError(f"unknown mode {mode!r}")
        if Hq % Hkv or N % blk or heads_per_chunk < 1:
            raise ValueError("need Hq % Hkv == 0, N % blk == 0 and heads_per_chunk >= 1")
        if mode == "gate" and (gate_thr is None or gate_thr.dtype != torch.float32 or seg != blk):
            raise ValueError("mode 'gate' lists every earlier block, so it needs seg == blk and gate_thr, "
                             "float32 [B, Hq, N / blk]")
        self.dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.shape = (B, Hq, Hkv, N, d)
        self.blk, self.seg, self.mode, self.dt = blk, seg, mode, density_or_tau
        self.band, self.n_sink, self.stop_tau = band, n_sink, stop_tau
        self.early = stop_tau > 0
        self.segmented = perm_per_segment
        self.G = Hq // Hkv
        nb, nseg = N // blk, (N + seg - 1) // seg
        bf = dict(dtype=torch.bfloat16, device=self.dev)
        self.Qd = torch.empty((B, Hq, N, d), **bf)
        self.Kd = torch.empty((B, Hkv, N, d), **bf)
        self.Vd = torch.empty((B, Hkv, N, d), **bf)
        self.Od = torch.empty((B, Hq, N, d), **bf)
        self.lse = torch.empty((B, Hq, N), dtype=torch.float32, device=self.dev)
        i32 = dict(dtype=torch.int32, device=self.dev)
        self.thr = gate_thr
        if mode in ("gate", "sample"):
            # natural key order for the attention
            self.perm = torch.arange(N, **i32).expand(B, Hkv, N).contiguous()
        else:
            self.perm = torch.empty((B, Hkv, nseg, N) if perm_per_segment else (B, Hkv, N), **i32)
        if mode == "gate":
            self.cap = max(nb - 1, 1)
            self.counts = torch.arange(nb, **i32).expand(B, Hq, nb).contiguous()
            self.idx = torch.arange(self.cap, **i32).expand(B, Hq, nb, self.cap).contiguous()
        else:
            self.cap = max(1, bd.select_capacity(N, blk, seg, mode, density_or_tau, band, n_sink))
            self.counts = torch.empty((B, Hq, nb), **i32)
            self.idx = torch.empty((B, Hq, nb, self.cap), **i32)
        self.units = [(b, lo, min(lo + heads_per_chunk, Hkv)) for b in range(B)
                      for lo in range(0, Hkv, heads_per_chunk)]
        # workspaces sized for the largest unit (the first one)
        b0, lo0, hi0 = self.units[0]
        q0, k0 = self._q(self.Qd, b0, lo0, hi0), self._k(self.Kd, b0, lo0, hi0)
        op_p = bd.PBS_OP_PERMUTE_SEGMENTED if perm_per_segment else bd.PBS_OP_PERMUTE
        op_s = (bd.PBS_OP_SELECT_SAMPLE if mode == "sample" else
                bd.PBS_OP_SELECT_SEGMENTED if perm_per_segment else bd.PBS_OP_SELECT)
        self.ws_p = self._ws(bd.workspace_size(op_p, q0, k0, blk, seg)) if mode in ("topk", "tau") else None
        self.ws_s = self._ws(bd.workspace_size(op_s, q0, k0, blk, seg)) if mode != "gate" else None
        self.s_in = torch.cuda.Stream(self.dev)
        self.s_cmp = torch.cuda.Stream(self.dev)
        self.s_out = torch.cuda.Stream(self.dev)
        n = len(self.units)
        self.ev_in = [torch.cuda.Event() for _ in range(n)]
        self.ev_cmp = [torch.cuda.Event() for _ in range(n)]
        self.ev_out = [torch.cuda.Event() for _ in range(n)]
        self._started = False

    # ---------------------------------------------------------------- views
    def _ws(self, nbytes: int) -> Optional[torch.Tensor]:
        return torch.empty(nbytes + 256, dtype=torch.uint8, device=self.dev) if nbytes else None

    def _q(self, t: torch.Tensor, b: int, lo: int, hi: int) -> torch.Tensor:
        return t[b:b + 1, lo * self.G:hi * self.G]

    @staticmethod
    def _k(t: torch.Tensor, b: int, lo: int, hi: int) -> torch.Tensor:
        return t[b:b + 1, lo:hi]

    def _check_host(self, name: str, t: torch.Tensor, H: int) -> None:
        B, _, _, N, d = self.shape
        if t.device.type != "cpu" or not t.is_pinned() or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous pinned bf16 host tensor")
        if tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {(B, H, N, d)}")

    # ----------------------------------------------------------------- run
    def run(self, Qh: torch.Tensor, Kh: torch.Tensor, Vh: torch.Tensor, Oh: torch.Tensor) -> None:
        """Enqueue one prefill and return.  Work already queued on the current
        stream comes first, and the current stream waits for the last copy of
        O, so synchronising it (or the device) makes ``Oh`` complete."""
        B, Hq, Hkv, N, d = self.shape
        for name, t, H in (("Q", Qh, Hq), ("K", Kh, Hkv), ("V", Vh, Hkv), ("O", Oh, Hq)):
            self._check_host(name, t, H)
        cur = torch.cuda.current_stream(self.dev)
        start = torch.cuda.Event()
        start.record(cur)
        for s in (self.s_in, self.s_cmp, self.s_out):
            s.wait_event(start)
        with torch.cuda.stream(self.s_in):
            for u, (b, lo, hi) in enumerate(self.units):
                if self._started:
                    # the previous prefill's kernels of this unit read these rows
                    self.s_in.wait_event(self.ev_cmp[u])
                self._q(self.Qd, b, lo, hi).copy_(self._q(Qh, b, lo, hi), non_blocking=True)
                self._k(self.Kd, b, lo, hi).copy_(self._k(Kh, b, lo, hi), non_blocking=True)
                self._k(self.Vd, b, lo, hi).copy_(self._k(Vh, b, lo, hi), non_blocking=True)
                self.ev_in[u].record(self.s_in)
        for u, (b, lo, hi) in enumerate(self.units):
            self.s_cmp.wait_event(self.ev_in[u])
            if self._started:
                # the previous prefill's copy of this unit's O is out
                self.s_cmp.wait_event(self.ev_out[u])
            self._compute(b, lo, hi)
            self.ev_cmp[u].record(self.s_cmp)
            self.s_out.wait_event(self.ev_cmp[u])
            with torch.cuda.stream(self.s_out):
                self._q(Oh, b, lo, hi).copy_(self._q(self.Od, b, lo, hi), non_blocking=True)
            self.ev_out[u].record(self.s_out)
        self._started = True
        cur.wait_event(self.ev_out[-1])

    def _compute(self, b: int, lo: int, hi: int) -> None:
        s = self.s_cmp
        Q, K, V = self._q(self.Qd, b, lo, hi), self._k(self.Kd, b, lo, hi), self._k(self.Vd, b, lo, hi)
        O, lse = self._q(self.Od, b, lo, hi), self._q(self.lse, b, lo, hi)
        perm = self._k(self.perm, b, lo, hi)
        counts, idx = self._q(self.counts, b, lo, hi), self._q(self.idx, b, lo, hi)
        if self.mode in ("topk", "tau"):
            permute = bd.pbs_permute_segmented if self.segmented else bd.pbs_permute
            permute(Q, K, self.blk, self.seg, self.n_sink, perm=perm, ws=self.ws_p, stream=s)
        if self.mode != "gate":
            bd.pbs_select(Q, K, None if self.mode == "sample" else perm, self.blk, self.seg, self.mode, self.dt,
                          self.band, self.n_sink, cap=self.cap, counts=counts, idx=idx, ws=self.ws_s, stream=s,
                          score_order=self.early)
        if self.early:
            bd.pbs_attn_fwd_early_stop(Q, K, V, perm, counts, idx, self.blk, self.seg, self.stop_tau, out=O,
                                       lse=lse, stream=s)
        else:
            thr = None if self.thr is None else self._q(self.thr, b, lo, hi)
            bd.pbs_attn_fwd(Q, K, V, perm, counts, idx, self.blk, self.seg, gate_thr=thr, out=O, lse=lse,
                            stream=s)
