"""Host-side plumbing for running PACE pools on several GPUs of one node.

Every (sequence, head) state is independent in both the decode step and the
period commit, so a multi-GPU deployment partitions sequences (pool slots)
across ranks and exchanges nothing on the data path.  What the ranks share is
bookkeeping: which global slots a rank owns, a barrier around timed regions,
and the slowest rank's time for throughput.  ``torch.distributed`` carries it
(NCCL on GPUs, gloo on CPU in tests).
"""
from __future__ import annotations

from typing import Tuple

__all__ = ["slot_range", "rank_of_slot", "barrier", "max_over_ranks", "aggregate_rate"]


def slot_range(global_slots: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced share ``[start, start + count)`` of ``global_slots``
    pool slots owned by ``rank`` of ``world``; the first ``global_slots % world``
    ranks take one extra slot.  Shares are disjoint and cover every slot."""
    if world < 1 or not (0 <= rank < world) or global_slots < 0:
        raise ValueError(f"bad partition: slots={global_slots} world={world} rank={rank}")
    base, extra = divmod(global_slots, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def rank_of_slot(slot: int, global_slots: int, world: int) -> int:
    """Inverse of :func:`slot_range`: the rank that owns global ``slot``."""
    if not (0 <= slot < global_slots):
        raise ValueError(f"slot {slot} outside [0, {global_slots})")
    base, extra = divmod(global_slots, world)
    big = extra * (base + 1)
    if slot < big:
        return slot // (base + 1)
    return extra + (slot - big) // base


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest ``x`` over all ranks (every rank gets it)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: int, world: int, max_elapsed_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (ranks start together after a barrier)."""
    if max_elapsed_ms <= 0:
        raise ValueError("elapsed time must be positive")
    return units_per_rank * world / (max_elapsed_ms * 1e-3)
