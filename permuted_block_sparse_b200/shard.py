"""How the path shards across GPUs (one process per GPU).

Permutation, selection and attention of different (batch, KV-head) groups
are independent: a KV head's permutation, its query heads' block lists and
their attention never read another group's data.  So the path shards with
no collective on the data path:

  * weak scaling: each rank runs its own problem (its own batch);
  * one problem over several GPUs: each rank takes a contiguous range of KV
    heads together with their query heads and writes its slice of O; the
    output is head-sharded, as in tensor-parallel attention (gathering O,
    if a caller wants it whole, is the caller's step).
"""
from __future__ import annotations

from typing import Tuple


def kv_head_range(Hkv: int, world: int, rank: int) -> Tuple[int, int]:
    """[lo, hi) of the KV heads rank `rank` of `world` processes: contiguous,
    disjoint, covering all heads, sizes differing by at most one."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(Hkv, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def query_head_range(Hq: int, Hkv: int, world: int, rank: int) -> Tuple[int, int]:
    """Query heads belonging to the rank's KV heads (Hq / Hkv per KV head)."""
    G = Hq // Hkv
    lo, hi = kv_head_range(Hkv, world, rank)
    return lo * G, hi * G


def seed_for_rank(seed: int, rank: int) -> int:
    """Seed of a rank's own synthetic problem under weak scaling."""
    return seed + rank


def max_over_ranks(values, dist=None):
    """Element-wise max of per-rank float values (all ranks get the result);
    without an initialised process group the local values are returned."""
    import torch
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return [float(v) for v in values]
    backend = dist.get_backend()
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]
