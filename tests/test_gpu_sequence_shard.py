"""The context-parallel form across devices (SequenceShardedInplace) with the library's kernels:
ranks emulated as threads of one process on one GPU, each with its own state and stream, whose
only exchange is the host-side hand-over of their delta sums (no kernel waits on another
rank's). The outputs of all ranks in token order and the final weight must match the oracle's
single scan, and a weight sum of ttt_add_f32 must be the fp32 sum bit for bit."""

import threading

import pytest
import torch

from gen import workloads
from oracle import inplace as oinp
from tests._util import rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


def test_add_f32_is_the_fp32_sum(cwl):
    g = torch.Generator().manual_seed(5)
    for n in (1, 7, 4096 + 3):
        y = torch.randn(n, generator=g).cuda()
        x = torch.randn(n, generator=g).cuda()
        want = y + x
        cwl.add_f32(y, x, 1.0)
        torch.cuda.synchronize()
        assert torch.equal(y, want)
    # Unaligned views take the scalar path.
    y = torch.randn(4099, generator=g).cuda()
    x = torch.randn(4099, generator=g).cuda()
    want = y[1:] - x[1:]
    cwl.add_f32(y[1:], x[1:].clone()[0:], -1.0)
    torch.cuda.synchronize()
    assert torch.equal(y[1:], want)


class _Exchange:
    """All-gather between threads: each puts its tensor, waits for the others, copies them all."""

    def __init__(self, world):
        self.world = world
        self.slots = [None] * world
        self.barrier = threading.Barrier(world, timeout=60)

    def for_rank(self, rank):
        def exchange(parts, mine):
            torch.cuda.current_stream().synchronize()
            self.slots[rank] = mine
            self.barrier.wait()
            for r in range(self.world):
                parts[r].copy_(self.slots[r])
            torch.cuda.current_stream().synchronize()
            self.barrier.wait()
        return exchange


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_sharded_threads(cwl, world):
    from chunked_weight_layers_b200.dist import SequenceShardedInplace
    C = 128
    calls = [2 * C * world, C * world]  # chunks a rank: 2, then 1
    T = sum(calls)
    spec = workloads.scaled(workloads.INPLACE_4B, T=T, C=C, d=256, f=384, seed=61 + world)
    x = workloads.inplace_inputs(spec, device="cuda")
    cfg = cwl.config("inplace", io_dtype=1, d_key=spec.f, d_val=spec.d, chunk=C, eta=spec.eta)
    ex = _Exchange(world)
    results, errors = {}, []

    def run(rank):
        try:
            torch.cuda.set_device(0)
            with torch.cuda.stream(torch.cuda.Stream()):
                layer = SequenceShardedInplace(cfg, x["W0"], exchange=ex.for_rank(rank), rank=rank, world=world)
                outs, t0 = [], 0
                for n in calls:
                    per = n // world
                    sl = slice(t0 + rank * per, t0 + (rank + 1) * per)
                    outs.append((sl, layer.scan(x["Z"][sl], x["Vhat"][sl])))
                    t0 += n
                torch.cuda.current_stream().synchronize()
                layer.state.poll()
                results[rank] = (outs, layer.get_weights())
        except BaseException as e:  # reported by the main thread
            errors.append(e)
            ex.barrier.abort()

    threads = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    O_ref, W_ref = oinp.inplace_scan(x["Z"].cpu(), x["Vhat"].cpu(), x["W0"].cpu(), spec.eta, C)
    O = torch.empty((T, spec.d), dtype=torch.bfloat16)
    for r in range(world):
        for sl, o in results[r][0]:
            O[sl] = o.cpu()
    eo = rel_err(O, O_ref)
    ew = max(rel_err(results[r][1], W_ref) for r in range(world))
    print(f"sequence-sharded over {world} thread ranks: O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL
    for r in range(1, world):
        assert torch.equal(results[r][1], results[0][1])
