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


def _inplace_worker(rank, world, port, out):
    """Rank ``rank`` scans its contiguous share of Wdown's rows (W0[rows], V̂[:, rows]) on its
    own, then the ranks all-gather their output columns; nothing else crosses ranks."""
    import numpy as np
    from oracle import inplace
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(7)
        T, C, d, f, eta = 96, 32, 10, 12, 0.05
        Z, V, W0 = rng.standard_normal((T, f)), rng.standard_normal((T, d)), 0.1 * rng.standard_normal((d, f))
        a, b = shard_range(d, rank, world)
        O_mine, W_mine = inplace.inplace_scan_rows(Z, V[:, a:b], W0[a:b], eta, C)
        cols = [torch.zeros(T, n, dtype=torch.float64) for n in
                (shard_range(d, r, world)[1] - shard_range(d, r, world)[0] for r in range(world))]
        dist.all_gather(cols, torch.from_numpy(np.ascontiguousarray(O_mine)))
        rows = [torch.zeros(n, f, dtype=torch.float64) for n in
                (shard_range(d, r, world)[1] - shard_range(d, r, world)[0] for r in range(world))]
        dist.all_gather(rows, torch.from_numpy(np.ascontiguousarray(W_mine)))
        O = torch.cat(cols, 1).numpy()
        W = torch.cat(rows, 0).numpy()
        O_ref, W_ref = inplace.inplace_scan(Z, V, W0, eta, C)
        out[rank] = bool(np.allclose(O, O_ref, rtol=0, atol=1e-12) and np.allclose(W, W_ref, rtol=0, atol=1e-12))
    finally:
        dist.destroy_process_group()


def test_inplace_rows_shard_across_two_gloo_ranks():
    """The In-Place scan shards over Wdown's rows: two ranks with half the rows each reproduce
    the single-process scan (to float64 rounding) after one all-gather of output columns."""
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
