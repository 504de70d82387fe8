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


class RowShardedInplace:
    """One In-Place layer whose Wdown rows are split over the ranks of a process group.

    Rank r owns rows [a, b) = shard_range(d_val, r, world) of Wdown [d_val, d_key]: its state
    holds W0[a:b], each scan reads the whole Z and the columns a:b of V̂ and produces the output
    columns O[:, a:b]. A row of the fast weight evolves on its own ("In-Place Test-Time
    Training", §2-§3: W_{c+1}[i] = W_c[i] + η·Σ_t V̂[t, i]·Z[t] needs only column i of V̂ and Z), so
    nothing crosses ranks inside the scan: one all-gather of output columns per call (and one
    of weight rows when the whole weight is read back) is the only exchange. The collectives are
    torch.distributed's (NCCL over NVLink on GPUs); no rank reads another's memory directly.

    ``make_state(cfg, W0_rows)`` builds the rank's state; by default the library's
    FastWeightState on the current CUDA device. Targets are given (target_mode 0): the fused
    target needs every input channel of X0 on every rank and is not sharded here.
    """

    def __init__(self, cfg, W0, group=None, make_state=None):
        import copy

        import torch.distributed as dist
        if getattr(cfg, "target_mode", 0) != 0:
            raise ValueError("RowShardedInplace shards In-Place layers with given targets (target_mode 0)")
        self.group = group
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.d = int(cfg.d_val)
        self.sizes = [b - a for a, b in (shard_range(self.d, r, self.world) for r in range(self.world))]
        self.rows = shard_range(self.d, self.rank, self.world)
        a, b = self.rows
        local = copy.copy(cfg)
        local.d_val = b - a
        if make_state is None:
            from . import FastWeightState
            make_state = FastWeightState
        self.state = make_state(local, W0[a:b].contiguous())

    def _gather(self, mine, dim):
        """All-gather ``mine`` (this rank's slice along ``dim``) into the full tensor, padding every
        slice to the largest rank's size so that the collective sees equal shapes."""
        import torch
        import torch.distributed as dist
        if self.world == 1:
            return mine
        width = max(self.sizes)
        shape = list(mine.shape)
        shape[dim] = width
        padded = torch.zeros(shape, dtype=mine.dtype, device=mine.device)
        padded.narrow(dim, 0, mine.shape[dim]).copy_(mine)
        parts = [torch.empty_like(padded) for _ in range(self.world)]
        dist.all_gather(parts, padded, group=self.group)
        return torch.cat([p.narrow(dim, 0, n) for p, n in zip(parts, self.sizes)], dim)

    def scan(self, Z, Vhat, T=None):
        """Continue the scan over T tokens: Z [T, d_key] and V̂ [T, d_val] whole on every rank.
        Returns the whole output O [T, d_val] on every rank."""
        import torch
        a, b = self.rows
        T = Z.shape[0] if T is None else T
        O_mine = torch.empty((T, b - a), dtype=Z.dtype, device=Z.device)
        self.state.chunk_scan(Z, Vhat[:, a:b].contiguous(), out=O_mine, T=T)
        return self._gather(O_mine, 1)

    def get_weights(self):
        """The whole fp32 weight [d_val, d_key], gathered from the ranks' rows."""
        import torch
        a, b = self.rows
        W_mine = torch.empty((b - a, self.state.cfg.d_key), dtype=torch.float32, device=self._device())
        self.state.get_weights(W_mine)
        return self._gather(W_mine, 0)

    def reset(self):
        self.state.reset()

    def _device(self):
        dev = getattr(self.state, "device", None)
        if dev is not None:
            return dev
        import torch
        return torch.device("cuda", torch.cuda.current_device())
