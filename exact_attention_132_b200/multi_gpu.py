"""Host-side plumbing for running the attention kernels on several GPUs.

Attention heads are independent: no (b, h) pair ever reads another head's Q, K
or V, in the forward or the backward.  So several GPUs split the heads (or the
batch) among themselves and each runs the single-GPU kernels on its share; there
is no data-path collective.  The only cross-rank communication is for timing
(max over ranks) and, optionally, gathering results.  One process per GPU.
"""
from __future__ import annotations


def shard_range(n_units: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous, balanced [start, stop) of `n_units` independent units for `rank`.

    The first n_units % world ranks get one extra unit; every unit is owned by
    exactly one rank.
    """
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} / world {world}")
    if n_units < 0:
        raise ValueError("n_units must be >= 0")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process group).

    Every rank must call this the same number of times, in the same order.
    """
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(flops_per_rank: float, steps: int, elapsed_ms: float, dist=None,
                         device=None) -> tuple[float, float]:
    """Whole-job TFLOP/s: all ranks' FLOPs divided by the slowest rank's time.

    Returns (tflops, max_elapsed_ms).
    """
    world = dist.get_world_size() if dist is not None and dist.is_initialized() else 1
    t = max_over_ranks(elapsed_ms, dist, device)
    return flops_per_rank * steps * world / (t * 1e-3) / 1e12, t
