"""ctypes binding of libpbs.so: argument marshalling only.

Every function here checks types, builds the C descriptors, allocates the
caller-side buffers the C ABI asks for (outputs, workspace) with torch, and
calls the library on torch's current CUDA stream.  All computation happens in
the library's sm_100a kernels; there is no fallback: if libpbs.so is missing
or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpbs.so")

PBS_OP_PERMUTE, PBS_OP_SELECT, PBS_OP_ATTN, PBS_OP_PERMUTE_SEGMENTED, PBS_OP_SELECT_SEGMENTED = 0, 1, 2, 3, 4
PBS_OP_SELECT_SAMPLE = 5
PBS_OP_PERMUTE_QUERIES = 6
PBS_SELECT_TOPK, PBS_SELECT_TAU, PBS_SELECT_SAMPLE = 0, 1, 2
_MODES = {"topk": PBS_SELECT_TOPK, "tau": PBS_SELECT_TAU, "sample": PBS_SELECT_SAMPLE}
PBS_SELECT_SCORE_ORDER, PBS_SELECT_PERM_PER_SEGMENT = 0x10, 0x20
PBS_ATTN_EARLY_STOP, PBS_ATTN_PERM_PER_SEGMENT, PBS_ATTN_CTA_PAIR = 1, 2, 4
STATUS = {0: "PBS_OK", -1: "PBS_ERR_INVALID_ARG", -2: "PBS_ERR_UNSUPPORTED", -3: "PBS_ERR_CAPACITY",
          -4: "PBS_ERR_CUDA", -5: "PBS_ERR_TIMEOUT", -6: "PBS_ERR_DEVICE_CHECK"}
EXPORTS = ("pbs_workspace_size", "pbs_permute", "pbs_permute_segmented", "pbs_select_capacity", "pbs_select",
           "pbs_attn_fwd", "pbs_attn_fwd_early_stop", "pbs_attn_fwd_ex", "pbs_check_device",
           "pbs_get_last_error", "pbs_version", "pbs_permute_noalloc", "pbs_test_inject_timeout",
           "pbs_permute_queries", "pbs_select_qperm", "pbs_attn_fwd_qperm")


class PbsError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class PbsTensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p),
                ("B", ctypes.c_int64), ("H", ctypes.c_int64), ("N", ctypes.c_int64), ("D", ctypes.c_int64),
                ("sB", ctypes.c_int64), ("sH", ctypes.c_int64), ("sN", ctypes.c_int64)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libpbs.so and declare its signatures (raises if missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libpbs.so not built at {path}; run python -m permuted_block_sparse_b200.build")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(PbsTensor)
    vp, i32, i64, dbl, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
    lib.pbs_workspace_size.argtypes = [i32, P, P, i32, i32]
    lib.pbs_workspace_size.restype = sz
    lib.pbs_permute.argtypes = [P, P, i32, i32, i32, vp, vp, sz, vp]
    lib.pbs_permute.restype = i32
    lib.pbs_permute_segmented.argtypes = [P, P, i32, i32, i32, vp, vp, sz, vp]
    lib.pbs_permute_segmented.restype = i32
    lib.pbs_attn_fwd_ex.argtypes = [P, P, P, vp, vp, vp, i32, i32, i32, ctypes.c_uint, vp, ctypes.c_float,
                                    ctypes.c_float, P, vp, vp, vp]
    lib.pbs_attn_fwd_ex.restype = i32
    lib.pbs_select_capacity.argtypes = [i64, i32, i32, i32, dbl, i32, i32]
    lib.pbs_select_capacity.restype = i32
    lib.pbs_select.argtypes = [P, P, vp, i32, i32, i32, dbl, i32, i32, vp, vp, i32, vp, sz, vp]
    lib.pbs_select.restype = i32
    lib.pbs_attn_fwd.argtypes = [P, P, P, vp, vp, vp, i32, i32, i32, vp, ctypes.c_float, P, vp, vp, vp, sz, vp]
    lib.pbs_attn_fwd.restype = i32
    lib.pbs_attn_fwd_early_stop.argtypes = [P, P, P, vp, vp, vp, i32, i32, i32, ctypes.c_float, ctypes.c_float,
                                            P, vp, vp, vp]
    lib.pbs_attn_fwd_early_stop.restype = i32
    lib.pbs_check_device.argtypes = [vp]
    lib.pbs_check_device.restype = i32
    lib.pbs_permute_queries.argtypes = [P, P, i32, i32, vp, vp, sz, vp]
    lib.pbs_permute_queries.restype = i32
    lib.pbs_select_qperm.argtypes = [P, P, vp, vp, i32, i32, i32, dbl, i32, vp, vp, i32, vp, sz, vp]
    lib.pbs_select_qperm.restype = i32
    lib.pbs_attn_fwd_qperm.argtypes = [P, P, P, vp, vp, vp, vp, i32, i32, i32, ctypes.c_float, P, vp, vp, vp]
    lib.pbs_attn_fwd_qperm.restype = i32
    lib.pbs_test_inject_timeout.argtypes = [ctypes.c_uint]
    lib.pbs_test_inject_timeout.restype = None
    lib.pbs_get_last_error.argtypes = []
    lib.pbs_get_last_error.restype = ctypes.c_char_p
    lib.pbs_version.argtypes = []
    lib.pbs_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(rc: int) -> None:
    if rc != 0:
        raise PbsError(rc, load().pbs_get_last_error().decode())


def describe(t: torch.Tensor) -> PbsTensor:
    """pbs_tensor for a [B, H, N, D] bf16 CUDA tensor with unit D stride."""
    if t.dim() != 4:
        raise ValueError("expected a [B, H, N, D] tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError("expected bfloat16")
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if t.stride(3) != 1:
        raise ValueError("the D dimension must be contiguous")
    B, H, N, D = t.shape
    sB, sH, sN, _ = t.stride()
    return PbsTensor(t.data_ptr(), B, H, N, D, sB, sH, sN)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _workspace(nbytes: int, device) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return None
    return torch.empty(nbytes + 256, dtype=torch.uint8, device=device)


def _aligned(ws: Optional[torch.Tensor]) -> Tuple[Optional[int], int]:
    if ws is None:
        return None, 0
    p = ws.data_ptr()
    a = (p + 255) & ~255
    return a, ws.numel() - (a - p)


def workspace_size(op: int, Q: torch.Tensor, K: torch.Tensor, blk: int, seg: int) -> int:
    q, k = describe(Q), describe(K)
    return load().pbs_workspace_size(op, ctypes.byref(q), ctypes.byref(k), blk, seg)


def select_capacity(N: int, blk: int, seg: int, mode: str, density_or_tau: float,
                    band: int = 0, n_sink: int = 0) -> int:
    if mode not in _MODES:
        raise ValueError(f"unknown selection mode {mode!r}; expected one of {sorted(_MODES)}")
    m = _MODES[mode]
    rc = load().pbs_select_capacity(N, blk, seg, m, float(density_or_tau), band, n_sink)
    _check(min(rc, 0))
    return rc


def pbs_permute(Q: torch.Tensor, K: torch.Tensor, blk: int, seg: int, n_sink: int = 0,
                perm: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """perm [B, Hkv, N] int32: per-segment stable descending sort of keys."""
    lib = load()
    q, k = describe(Q), describe(K)
    B, Hkv, N, _ = K.shape
    if perm is None:
        perm = torch.empty((B, Hkv, N), dtype=torch.int32, device=K.device)
    if ws is None:
        ws = _workspace(lib.pbs_workspace_size(PBS_OP_PERMUTE, ctypes.byref(q), ctypes.byref(k), blk, seg), K.device)
    wp, wn = _aligned(ws)
    _check(lib.pbs_permute(ctypes.byref(q), ctypes.byref(k), blk, seg, n_sink, perm.data_ptr(), wp, wn,
                           _stream(stream)))
    return perm


def pbs_permute_segmented(Q: torch.Tensor, K: torch.Tensor, blk: int, seg: int, n_sink: int = 0,
                          perm: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """perm [B, Hkv, nseg, N] int32: one permutation per query segment (its
    history's key segments sorted by the segment's pooled query)."""
    lib = load()
    q, k = describe(Q), describe(K)
    B, Hkv, N, _ = K.shape
    nseg = (N + seg - 1) // seg
    if perm is None:
        perm = torch.empty((B, Hkv, nseg, N), dtype=torch.int32, device=K.device)
    if ws is None:
        ws = _workspace(lib.pbs_workspace_size(PBS_OP_PERMUTE_SEGMENTED, ctypes.byref(q), ctypes.byref(k), blk, seg),
                        K.device)
    wp, wn = _aligned(ws)
    _check(lib.pbs_permute_segmented(ctypes.byref(q), ctypes.byref(k), blk, seg, n_sink, perm.data_ptr(), wp, wn,
                                     _stream(stream)))
    return perm


def pbs_select(Q: torch.Tensor, K: torch.Tensor, perm: torch.Tensor, blk: int, seg: int,
               mode: str = "topk", density_or_tau: float = 1.0, band: int = 0, n_sink: int = 0,
               cap: Optional[int] = None, counts: Optional[torch.Tensor] = None,
               idx: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
               stream=None, score_order: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """(counts [B, Hq, nb] int32, idx [B, Hq, nb, cap] int32) block lists,
    ascending, or in visiting order (forced blocks, then descending block
    score) with ``score_order``."""
    lib = load()
    q, k = describe(Q), describe(K)
    B, Hq, N, _ = Q.shape
    nb = N // blk
    if mode not in _MODES:
        raise ValueError(f"unknown selection mode {mode!r}; expected one of {sorted(_MODES)}")
    m = _MODES[mode]
    if score_order:
        m |= PBS_SELECT_SCORE_ORDER
    op = PBS_OP_SELECT_SAMPLE if mode == "sample" else PBS_OP_SELECT
    if perm is not None and perm.dim() == 4:   # one permutation per query segment
        m |= PBS_SELECT_PERM_PER_SEGMENT
        op = PBS_OP_SELECT_SEGMENTED
    if cap is None:
        cap = max(1, select_capacity(N, blk, seg, mode, density_or_tau, band, n_sink))
    if counts is None:
        counts = torch.empty((B, Hq, nb), dtype=torch.int32, device=Q.device)
    if idx is None:
        idx = torch.empty((B, Hq, nb, cap), dtype=torch.int32, device=Q.device)
    if ws is None:
        ws = _workspace(lib.pbs_workspace_size(op, ctypes.byref(q), ctypes.byref(k), blk, seg), Q.device)
    wp, wn = _aligned(ws)
    _check(lib.pbs_select(ctypes.byref(q), ctypes.byref(k), _ptr(perm), blk, seg, m, float(density_or_tau),
                          band, n_sink, counts.data_ptr(), idx.data_ptr(), cap, wp, wn, _stream(stream)))
    return counts, idx


def pbs_attn_fwd(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, perm: torch.Tensor,
                 counts: torch.Tensor, idx: torch.Tensor, blk: int, seg: int,
                 gate_thr: Optional[torch.Tensor] = None, softmax_scale: Optional[float] = None,
                 out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                 want_lse: bool = True, stats: Optional[torch.Tensor] = None,
                 stream=None, cta_pair: bool = False) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """(O [B, Hq, N, D] bf16, LSE [B, Hq, N] fp32 or None).  ``cta_pair``
    runs the CTA-pair kernel where it applies (d = blk = 128, query heads per
    KV head a multiple of 4, no gate); its results are the same."""
    lib = load()
    B, Hq, N, D = Q.shape
    if out is None:
        out = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=Q.device)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if gate_thr is not None and gate_thr.dtype != torch.float32:
        raise TypeError("gate_thr must be float32")
    if stats is not None and stats.dtype != torch.int64:
        raise TypeError("stats must be int64")
    q, k, v, o = describe(Q), describe(K), describe(V), describe(out)
    flags = (PBS_ATTN_PERM_PER_SEGMENT if perm.dim() == 4 else 0) | (PBS_ATTN_CTA_PAIR if cta_pair else 0)
    if flags:                                # one permutation per query segment / one-CTA kernel
        _check(lib.pbs_attn_fwd_ex(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), perm.data_ptr(),
                                   counts.data_ptr(), idx.data_ptr(), idx.shape[-1], blk, seg,
                                   flags, _ptr(gate_thr), 0.0, float(softmax_scale),
                                   ctypes.byref(o), _ptr(lse), _ptr(stats), _stream(stream)))
        return out, lse
    _check(lib.pbs_attn_fwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), perm.data_ptr(),
                            counts.data_ptr(), idx.data_ptr(), idx.shape[-1], blk, seg, _ptr(gate_thr),
                            float(softmax_scale), ctypes.byref(o), _ptr(lse), _ptr(stats), None, 0,
                            _stream(stream)))
    return out, lse


def pbs_permute_queries(Q: torch.Tensor, K: torch.Tensor, blk: int, seg: int,
                        qperm: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """qperm [B, Hq, N] int32: S2O's query permutation (per segment, queries
    by descending score against the KV head's guide vector)."""
    lib = load()
    q, k = describe(Q), describe(K)
    B, Hq, N, _ = Q.shape
    if qperm is None:
        qperm = torch.empty((B, Hq, N), dtype=torch.int32, device=Q.device)
    if ws is None:
        ws = _workspace(lib.pbs_workspace_size(PBS_OP_PERMUTE_QUERIES, ctypes.byref(q), ctypes.byref(k), blk, seg),
                        Q.device)
    wp, wn = _aligned(ws)
    _check(lib.pbs_permute_queries(ctypes.byref(q), ctypes.byref(k), blk, seg, qperm.data_ptr(), wp, wn,
                                   _stream(stream)))
    return qperm


def pbs_select_qperm(Q: torch.Tensor, K: torch.Tensor, perm: torch.Tensor, qperm: torch.Tensor, blk: int,
                     seg: int, mode: str = "topk", density_or_tau: float = 1.0, n_sink: int = 0,
                     cap: Optional[int] = None, counts: Optional[torch.Tensor] = None,
                     idx: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                     stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(counts, idx) block lists of the permuted query blocks (ascending)."""
    lib = load()
    q, k = describe(Q), describe(K)
    B, Hq, N, _ = Q.shape
    nb = N // blk
    if mode not in ("topk", "tau"):
        raise ValueError(f"permuted queries take mode 'topk' or 'tau', not {mode!r}")
    if cap is None:
        cap = max(1, select_capacity(N, blk, seg, mode, density_or_tau, 0, n_sink))
    if counts is None:
        counts = torch.empty((B, Hq, nb), dtype=torch.int32, device=Q.device)
    if idx is None:
        idx = torch.empty((B, Hq, nb, cap), dtype=torch.int32, device=Q.device)
    if ws is None:
        ws = _workspace(lib.pbs_workspace_size(PBS_OP_SELECT, ctypes.byref(q), ctypes.byref(k), blk, seg), Q.device)
    wp, wn = _aligned(ws)
    _check(lib.pbs_select_qperm(ctypes.byref(q), ctypes.byref(k), perm.data_ptr(), qperm.data_ptr(), blk, seg,
                                _MODES[mode], float(density_or_tau), n_sink, counts.data_ptr(), idx.data_ptr(), cap,
                                wp, wn, _stream(stream)))
    return counts, idx


def pbs_attn_fwd_qperm(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, perm: torch.Tensor,
                       qperm: torch.Tensor, counts: torch.Tensor, idx: torch.Tensor, blk: int, seg: int,
                       softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                       stats: Optional[torch.Tensor] = None,
                       stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """(O, LSE) at the queries' original positions, for lists indexed by
    permuted query block."""
    lib = load()
    B, Hq, N, D = Q.shape
    if out is None:
        out = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=Q.device)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if stats is not None and stats.dtype != torch.int64:
        raise TypeError("stats must be int64")
    q, k, v, o = describe(Q), describe(K), describe(V), describe(out)
    _check(lib.pbs_attn_fwd_qperm(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), perm.data_ptr(),
                                  qperm.data_ptr(), counts.data_ptr(), idx.data_ptr(), idx.shape[-1], blk, seg,
                                  float(softmax_scale), ctypes.byref(o), _ptr(lse), _ptr(stats), _stream(stream)))
    return out, lse


def pbs_attn_fwd_early_stop(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, perm: torch.Tensor,
                            counts: torch.Tensor, idx: torch.Tensor, blk: int, seg: int, stop_tau: float,
                            softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                            lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                            stats: Optional[torch.Tensor] = None,
                            stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """(O, LSE): S2O's two passes with the early-stopping rule; ``idx`` holds
    each block's list in visiting order."""
    lib = load()
    B, Hq, N, D = Q.shape
    if out is None:
        out = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=Q.device)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if stats is not None and stats.dtype != torch.int64:
        raise TypeError("stats must be int64")
    q, k, v, o = describe(Q), describe(K), describe(V), describe(out)
    if perm.dim() == 4:                      # one permutation per query segment
        _check(lib.pbs_attn_fwd_ex(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), perm.data_ptr(),
                                   counts.data_ptr(), idx.data_ptr(), idx.shape[-1], blk, seg,
                                   PBS_ATTN_EARLY_STOP | PBS_ATTN_PERM_PER_SEGMENT, None, float(stop_tau),
                                   float(softmax_scale), ctypes.byref(o), _ptr(lse), _ptr(stats),
                                   _stream(stream)))
        return out, lse
    _check(lib.pbs_attn_fwd_early_stop(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), perm.data_ptr(),
                                       counts.data_ptr(), idx.data_ptr(), idx.shape[-1], blk, seg,
                                       float(stop_tau), float(softmax_scale), ctypes.byref(o), _ptr(lse),
                                       _ptr(stats), _stream(stream)))
    return out, lse


def pbs_check_device(stream=None) -> None:
    """Synchronise and raise if a device-side check or bounded wait failed."""
    _check(load().pbs_check_device(_stream(stream)))


def test_inject_timeout(limit_polls: int) -> None:
    """Failure-path test hook (see pbs.h): > 0 makes later attention launches
    time out on purpose (bounded waits, no fault); 0 turns it off."""
    load().pbs_test_inject_timeout(int(limit_polls))


def version() -> str:
    return load().pbs_version().decode()
