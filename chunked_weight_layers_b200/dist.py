"""Host-side plumbing for running the scan on several GPUs of one node, one process per GPU.

The scan shards without a data-path collective: (sequence, head) problems are independent
for TTT-Linear and the gate, and Wdown rows are independent for In-Place. Each rank takes a
contiguous share of the units; the only collective is one all-reduce of the timing scalar
(max over ranks) at the end of a measurement.
"""

from __future__ import annotations


def shard_range(n_units: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous share [start, stop) of ``n_units`` for ``rank`` of ``world`` (sizes differ by ≤ 1)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    if n_units < 0:
        raise ValueError("n_units must be non-negative")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Max of ``value`` over all ranks of the default process group (the value itself without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
