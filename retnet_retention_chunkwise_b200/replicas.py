"""Host-side logic for running the retention calls on several GPUs.

Heads and batch rows are independent (page "Retentive Networks -- Microsoft
...", section "Il meccanismo": one gamma per head, no mixing between heads), so
the work shards over (batch, head) pairs with no exchange between GPUs: each
rank owns a contiguous range of pairs, or, for weak scaling, a full replica of
the per-GPU workload.  The only collectives are the timing reductions
(max over ranks) and the token count (sum over ranks).  Everything here works
with any torch.distributed backend; the tests run it with gloo on the CPU.
"""
from __future__ import annotations

import torch


def shard_pairs(n_pairs: int, rank: int, world: int):
    """Contiguous [begin, end) range of (batch, head) pairs owned by `rank`.

    The ranges of all ranks partition [0, n_pairs) and differ in size by at most one."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("bad rank/world")
    base, extra = divmod(n_pairs, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def _reduce(x: float, op, group=None, device="cpu") -> float:
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op, group=group)
    return float(t.item())


def max_over_ranks(x: float, group=None, device="cpu") -> float:
    import torch.distributed as dist
    return _reduce(x, dist.ReduceOp.MAX if dist.is_available() else None, group, device)


def sum_over_ranks(x: float, group=None, device="cpu") -> float:
    import torch.distributed as dist
    return _reduce(x, dist.ReduceOp.SUM if dist.is_available() else None, group, device)


def job_throughput(units_local: float, seconds_local: float, group=None, device="cpu"):
    """Whole-job throughput: units summed over ranks / time maxed over ranks.

    Returns (units_per_second, total_units, max_seconds)."""
    total = sum_over_ranks(units_local, group, device)
    t = max_over_ranks(seconds_local, group, device)
    return (total / t if t > 0 else float("nan")), total, t
