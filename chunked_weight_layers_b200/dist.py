"""Host-side plumbing for running the scan on several GPUs of one node, one process per GPU.

The scan shards without a data-path collective: (sequence, head) problems are independent
for TTT-Linear and the gate, and Wdown rows are independent for In-Place. Each rank takes a
contiguous share of the units; the only collective is one all-reduce of the timing scalar
(max over ranks) at the end of a measurement. Two helpers split one In-Place layer instead:
by Wdown rows (an all-gather of output columns a call) and by the sequence (the
context-parallel form: an all-gather of the ranks' delta sums a call).
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


class SequenceShardedInplace:
    """One In-Place layer whose sequence is split over the ranks of a process group: the
    context-parallel form across devices ("In-Place Test-Time Training", §6, context
    parallelism: the chunk deltas, an exclusive prefix sum of them, then every chunk's apply).

    Rank r scans its own contiguous run of whole chunks (the ranks in token order). The update
    η·V̂_cᵀ·Z_c does not depend on the weight, so a first scan of the rank's chunks from a zero
    weight leaves exactly the sum S_r of its deltas; the ranks all-gather those sums, rank r
    starts its real scan from W + Σ_{r' < r} S_r' (W: the weight before this call), and every
    rank ends holding W + Σ_r' S_r', the weight after the whole sequence, so the next call
    continues the scan. The sums are formed by the library (``ttt_add_f32``); the all-gather is
    torch.distributed's (NCCL over NVLink on GPUs; no rank reads another's memory directly).
    Each rank scans its tokens twice: on N ranks a call costs about 2/N of one device's scan
    plus the exchange of N fp32 weights.

    ``make_state(cfg, W0)`` builds the rank's state and ``add(y, x, alpha)`` forms y += alpha·x
    (by default the library's FastWeightState on the current CUDA device and ``add_f32``);
    ``exchange(parts, mine)``, with ``rank`` and ``world``, replaces the process group's
    all-gather (by default torch.distributed's over ``group``). Targets are given (target_mode 0).
    """

    def __init__(self, cfg, W0, group=None, make_state=None, add=None, exchange=None, rank=None, world=None):
        import torch.distributed as dist
        if getattr(cfg, "target_mode", 0) != 0:
            raise ValueError("SequenceShardedInplace shards In-Place layers with given targets (target_mode 0)")
        self.group = group
        if exchange is None:
            self.rank = dist.get_rank(group) if dist.is_initialized() else 0
            self.world = dist.get_world_size(group) if dist.is_initialized() else 1
            exchange = lambda parts, mine: dist.all_gather(parts, mine, group=group)  # noqa: E731
        else:
            self.rank, self.world = int(rank), int(world)
        self.exchange = exchange
        if make_state is None or add is None:
            from . import FastWeightState, add_f32
            make_state = make_state or FastWeightState
            add = add or add_f32
        self.add = add
        self.W0 = W0.clone()
        self.W = W0.clone()          # the weight before the next call, the same on every rank
        self.state = make_state(cfg, W0)

    def scan(self, Z, Vhat, T=None):
        """This rank's tokens: Z [T_r, d_key], V̂ [T_r, d_val], T_r a multiple of the chunk (the
        ranks' runs laid end to end in rank order form the sequence). Returns O [T_r, d_val]."""
        import torch
        T = Z.shape[0] if T is None else T
        O = torch.empty((T, self.W.shape[0]), dtype=Z.dtype, device=Z.device)
        if self.world > 1:
            self.state.set_weights(torch.zeros_like(self.W))
            self.state.chunk_scan(Z, Vhat, out=O, T=T)       # outputs discarded: the weight is S_r
            S = torch.empty_like(self.W)
            self.state.get_weights(S)
            parts = [torch.empty_like(S) for _ in range(self.world)]
            self.exchange(parts, S)
        else:
            parts = []
        start = self.W.clone()
        for p in parts[:self.rank]:
            self.add(start, p, 1.0)
        self.state.set_weights(start)
        self.state.chunk_scan(Z, Vhat, out=O, T=T)
        if self.world > 1:
            end = start.clone()
            for p in parts[self.rank:]:
                self.add(end, p, 1.0)
            self.state.set_weights(end)
        else:
            end = torch.empty_like(self.W)
            self.state.get_weights(end)
        self.W = end
        return O

    def get_weights(self):
        """The fp32 weight after the last call's whole sequence [d_val, d_key] (every rank)."""
        return self.W.clone()

    def reset(self):
        self.W = self.W0.clone()
        self.state.reset()
