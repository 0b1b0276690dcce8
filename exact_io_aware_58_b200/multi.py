"""Host-side logic for running the attention path on several GPUs.

Every (batch, head) pair is an independent problem: the forward and the
backward of one head never read another head's data ("Attention and KV
Compression", section "The composability point": the kernel tiles over
whatever heads exist).  So work is split across ranks by whole heads (or whole
batches) with no collective on the data path; the only communication is the
timing reduction (max over ranks) and, optionally, gathering results for a
check.  One process per GPU, launched by torchrun.
"""

from __future__ import annotations

import torch


def shard_range(total: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous [start, stop) share of ``total`` units for ``rank``: sizes
    differ by at most one, lower ranks take the larger shares."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("bad world/rank")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of the batch a rank draws when each rank runs its own batch (weak scaling)."""
    return base_seed + rank


def max_over_ranks(values, device=None, group=None) -> list[float]:
    """Element-wise max of per-rank floats (e.g. elapsed milliseconds)."""
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return [float(x) for x in t.tolist()]


def aggregate_tflops(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's FLOPs over the slowest rank's time."""
    return flops_per_rank * world / (ms_max * 1e-3) / 1e12
