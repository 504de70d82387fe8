"""The multi-rank host logic on CPU: two gloo ranks split the units with no gap or overlap and
agree on the max-over-ranks time."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from chunked_weight_layers_b200.dist import max_over_ranks, shard_range


def test_shard_range_covers_units():
    for n in (0, 1, 7, 96, 97, 1000):
        for world in (1, 2, 3, 8):
            got = [shard_range(n, r, world) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == n
            assert all(got[i][1] == got[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a, b = shard_range(96, rank, world)
        mine = torch.arange(a, b, dtype=torch.int64)
        sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sizes, torch.tensor([b - a]))
        gathered = [torch.zeros(int(s.item()), dtype=torch.int64) for s in sizes]
        dist.all_gather(gathered, mine)
        units = torch.cat(gathered)
        t = max_over_ranks(1.5 + rank)
        out[rank] = (sorted(units.tolist()) == list(range(96)), t)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        assert out[0] == (True, 2.5) and out[1] == (True, 2.5)


class _OracleState:
    """Stand-in for the library's state in this CPU test: the oracle's scan of a row block,
    behind the calls RowShardedInplace makes (chunk_scan, get_weights, reset)."""

    device = torch.device("cpu")

    def __init__(self, cfg, W0_rows):
        self.cfg = cfg
        self.W0 = W0_rows.clone()
        self.W = W0_rows.clone()

    def chunk_scan(self, Z, Vhat, out, T):
        from oracle import inplace
        O, W = inplace.inplace_scan_rows(Z[:T].numpy(), Vhat[:T].numpy(), self.W.numpy(), self.cfg.eta, self.cfg.chunk)
        out.copy_(torch.from_numpy(O))
        self.W = torch.from_numpy(W)

    def get_weights(self, W):
        W.copy_(self.W)

    def reset(self):
        self.W = self.W0.clone()


def _inplace_worker(rank, world, port, out):
    """Each rank runs RowShardedInplace (the product's host logic: row shares, V̂ column slices,
    padded all-gathers) over the oracle's row scan; the gathered O and W must equal the
    single-process scan, over two calls in a row."""
    import numpy as np
    import chunked_weight_layers_b200 as cwl
    from chunked_weight_layers_b200.dist import RowShardedInplace
    from oracle import inplace
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(7)
        T, C, d, f, eta = 96, 32, 11, 12, 0.05
        Z, V, W0 = rng.standard_normal((T, f)), rng.standard_normal((T, d)), 0.1 * rng.standard_normal((d, f))
        cfg = cwl.abi.ttt_config()
        cfg.rule, cfg.io_dtype, cfg.d_key, cfg.d_val, cfg.chunk, cfg.eta = 0, 0, f, d, C, eta
        layer = RowShardedInplace(cfg, torch.from_numpy(W0), make_state=_OracleState)
        Zt, Vt = torch.from_numpy(Z), torch.from_numpy(V)
        O1 = layer.scan(Zt[:64], Vt[:64])
        O2 = layer.scan(Zt[64:], Vt[64:])
        W = layer.get_weights().numpy()
        O = torch.cat([O1, O2]).numpy()
        O_ref, W_ref = inplace.inplace_scan(Z, V, W0, cfg.eta, C)  # η as the config holds it (fp32)
        # The weight is read back as fp32, like the library's state.
        ok = np.allclose(O, O_ref, rtol=0, atol=1e-12) and np.array_equal(W, W_ref.astype(np.float32))
        ok = ok and layer.rows == shard_range(d, rank, world) and layer.state.W.shape[0] == layer.rows[1] - layer.rows[0]
        layer.reset()
        ok = ok and np.array_equal(layer.get_weights().numpy(), W0.astype(np.float32))
        out[rank] = bool(ok)
    finally:
        dist.destroy_process_group()


def test_inplace_rows_shard_across_two_gloo_ranks():
    """The In-Place scan shards over Wdown's rows: two ranks (11 rows: 6 and 5) each holding their
    rows reproduce the single-process scan (to float64 rounding) after one all-gather of output
    columns a call."""
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_inplace_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        assert out[0] is True and out[1] is True


class _OracleWholeState(_OracleState):
    """The oracle's scan of the whole weight, with set_weights (the calls SequenceShardedInplace
    makes)."""

    def chunk_scan(self, Z, Vhat, out, T):
        from oracle import inplace
        O, W = inplace.inplace_scan(Z[:T].numpy(), Vhat[:T].numpy(), self.W.numpy(), self.cfg.eta, self.cfg.chunk)
        out.copy_(torch.from_numpy(O))
        self.W = torch.from_numpy(W)

    def set_weights(self, W):
        self.W = W.clone()


def _add(y, x, alpha):
    y.add_(x, alpha=alpha)
    return y


def _sequence_worker(rank, world, port, out):
    """Each rank runs SequenceShardedInplace (the product's host logic: a first scan from zero
    for the rank's delta sum, the all-gather, the rank's start and end weights) over the oracle's
    scan, on its own run of chunks; the outputs of all ranks in token order and the final weight
    must be the single-process scan's, over two calls in a row."""
    import numpy as np
    import chunked_weight_layers_b200 as cwl
    from chunked_weight_layers_b200.dist import SequenceShardedInplace
    from oracle import inplace
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(11)
        C, d, f, eta = 32, 7, 9, 0.05
        calls = [96 * world, 32 * world]  # tokens of each call: 3 chunks a rank, then 1
        T = sum(calls)
        Z, V, W0 = rng.standard_normal((T, f)), rng.standard_normal((T, d)), 0.1 * rng.standard_normal((d, f))
        cfg = cwl.abi.ttt_config()
        cfg.rule, cfg.io_dtype, cfg.d_key, cfg.d_val, cfg.chunk, cfg.eta = 0, 0, f, d, C, eta
        layer = SequenceShardedInplace(cfg, torch.from_numpy(W0), make_state=_OracleWholeState, add=_add)
        Zt, Vt = torch.from_numpy(Z), torch.from_numpy(V)
        mine, t0 = [], 0
        for n in calls:
            a, b = shard_range(n // C, rank, world)
            sl = slice(t0 + a * C, t0 + b * C)
            mine.append((sl, layer.scan(Zt[sl], Vt[sl])))
            t0 += n
        O_ref, W_ref = inplace.inplace_scan(Z, V, W0, cfg.eta, C)
        ok = all(np.allclose(o.numpy(), O_ref[sl], rtol=0, atol=1e-12) for sl, o in mine)
        ok = ok and np.allclose(layer.get_weights().numpy(), W_ref, rtol=0, atol=1e-12)
        # Without the exchange every rank after the first would start from W0.
        if rank > 0:
            O_alone, _ = inplace.inplace_scan(Z[mine[0][0]], V[mine[0][0]], W0, cfg.eta, C)
            ok = ok and not np.allclose(O_alone, mine[0][1].numpy())
        layer.reset()
        ok = ok and np.array_equal(layer.get_weights().numpy(), W0)
        out[rank] = bool(ok)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_inplace_sequence_shards_across_gloo_ranks(world):
    """The context-parallel form across ranks: each rank scans its own chunks of the sequence and
    the ranks exchange their delta sums once a call; the outputs in token order and the final
    weight equal the single-process scan (to float64 rounding)."""
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_sequence_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        assert all(out[r] is True for r in range(world))
