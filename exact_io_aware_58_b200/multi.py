"""Host-side logic for running the attention path on several GPUs.

Every (batch, head) pair is an independent problem: the forward and the
backward of one head never read another head's data ("Attention and KV
Compression", section "The composability point": the kernel tiles over
whatever heads exist).  So work is split across ranks by whole heads (or whole
batches) with no collective on the data path; the only communication is the
timing reduction (max over ranks) and, optionally, gathering results for a
check.  One process per GPU.

The benchmark's per-rank loop lives here (``run_timed``) with the clock and
the barrier passed in, so the same code runs with CUDA events on a GPU and
with a host clock in the multi-process CPU tests.
"""

from __future__ import annotations

import os

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


class CudaClock:
    """Timestamps as CUDA events recorded on one stream (the stream the
    kernels are launched on); ``sync`` waits for the device."""

    def __init__(self, stream):
        self.stream = stream

    def mark(self):
        e = torch.cuda.Event(enable_timing=True)
        e.record(self.stream)
        return e

    @staticmethod
    def elapsed_ms(a, b) -> float:
        return a.elapsed_time(b)

    @staticmethod
    def sync():
        torch.cuda.synchronize()


def run_timed(step, steps: int, warmup: int, clock, barrier=None, n_segments: int = 1, on_timed_start=None):
    """``warmup`` untimed calls of ``step(mark)``, then a barrier and a sync on
    both sides of ``steps`` timed calls.  ``step`` calls ``mark()`` between its
    kernels: ``n_segments`` segments need ``n_segments - 1`` inner marks (the
    first and last are taken here).  Returns (total ms of the timed region,
    [mean ms of each segment]) for this rank; reduce them with
    ``max_over_ranks``."""
    for _ in range(warmup):
        step(lambda: None)
    if barrier is not None:
        barrier()
    clock.sync()
    if on_timed_start is not None:
        on_timed_start()
    marks = []
    t0 = clock.mark()
    for _ in range(steps):
        m = [clock.mark()]
        step(lambda: m.append(clock.mark()))
        m.append(clock.mark())
        if len(m) != n_segments + 1:
            raise RuntimeError(f"step made {len(m) - 2} inner marks, expected {n_segments - 1}")
        marks.append(m)
    t1 = clock.mark()
    clock.sync()
    if barrier is not None:
        barrier()
    total = clock.elapsed_ms(t0, t1)
    seg = [sum(clock.elapsed_ms(m[k], m[k + 1]) for m in marks) / steps for k in range(n_segments)]
    return total, seg


def rank_envs(n: int, port: int, base_env=None) -> list[dict]:
    """Environment of each of ``n`` rank processes on this node (one GPU each):
    the torch.distributed variables the benchmark reads."""
    envs = []
    for r in range(n):
        e = dict(os.environ if base_env is None else base_env)
        e.update({"RANK": str(r), "LOCAL_RANK": str(r), "WORLD_SIZE": str(n), "LOCAL_WORLD_SIZE": str(n),
                  "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
        envs.append(e)
    return envs
