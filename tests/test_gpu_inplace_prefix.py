"""GPU parity of the context-parallel In-Place form (TTT_OPT_INPLACE_PREFIX): all chunk deltas,
their exclusive prefix sums, then all chunk outputs ("In-Place Test-Time Training", §6),
against the oracle's prefix form and its sequential scan."""

import numpy as np
import pytest
import torch

from gen import workloads
from oracle import inplace as ora
from tests._util import bf16_round, rel_err, to_np

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


def scan(cwl, x, C, eta, prefix=True, calls=1):
    Z, V = x["Z"], x["Vhat"]
    T = Z.shape[0]
    d, f = x["W0"].shape
    st = cwl.FastWeightState(cwl.config("inplace", io_dtype=1, d_key=f, d_val=d, chunk=C, eta=eta), x["W0"])
    if prefix:
        st.set_option(cwl.abi.TTT_OPT_INPLACE_PREFIX, 1)
    O = torch.empty((T, d), device="cuda", dtype=torch.bfloat16)
    step = T // calls
    for a in range(0, T, step):
        st.chunk_scan(Z[a:a + step], V[a:a + step], out=O[a:a + step])
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    st.poll()
    return O, W, st


def test_exact_integers_bit_exact(cwl):
    """Sparse {-1,0,1} inputs, W0 in steps of 1/64, η = 2^-6: every delta, prefix sum and weight
    is exact, so O equals bf16(oracle) and the final W equals the oracle's bit for bit."""
    g = torch.Generator().manual_seed(19)
    T, C, d, f = 512, 128, 136, 200

    def sparse(shape, p):
        v = torch.randint(-1, 2, shape, generator=g).float()
        return v * (torch.rand(shape, generator=g) < p)

    Z, V = sparse((T, f), 0.15), sparse((T, d), 0.15)
    W0 = torch.randint(-32, 33, (d, f), generator=g).float() / 64
    O_ref, W_ref = ora.inplace_scan_prefix(Z, V, W0, 2.0 ** -6, C)
    x = {"Z": Z.to(torch.bfloat16).cuda(), "Vhat": V.to(torch.bfloat16).cuda(), "W0": W0.cuda()}
    O, W, _ = scan(cwl, x, C, 2.0 ** -6)
    assert np.array_equal(to_np(O), bf16_round(O_ref))
    assert np.array_equal(to_np(W), W_ref)


@pytest.mark.parametrize("d,f,T", [(256, 256, 512), (200, 328, 640), (392, 520, 384)])
def test_small_random(cwl, d, f, T):
    """Random inputs, tile-ragged widths: against the oracle's prefix form and the sequential
    oracle, and against the GPU's sequential form."""
    spec = workloads.scaled(workloads.INPLACE_4B, T=T, C=128, d=d, f=f, seed=131 + d)
    x = workloads.inplace_inputs(spec, device="cuda")
    O, W, _ = scan(cwl, x, spec.C, spec.eta)
    Zc, Vc, W0c = x["Z"].cpu(), x["Vhat"].cpu(), x["W0"].cpu()
    Op, Wp = ora.inplace_scan_prefix(Zc, Vc, W0c, spec.eta, spec.C)
    Os, Ws = ora.inplace_scan(Zc, Vc, W0c, spec.eta, spec.C)
    eo, ew = rel_err(O, Op), rel_err(W, Wp)
    print(f"context-parallel d={d} f={f} T={T}: O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL
    assert rel_err(O, Os) <= TOL and rel_err(W, Ws) <= TOL
    O2, W2, _ = scan(cwl, x, spec.C, spec.eta, prefix=False)
    assert rel_err(O, O2.float()) <= TOL and rel_err(W, W2) <= 1e-5


def test_streaming_and_switching_forms(cwl):
    """Two context-parallel calls, then a sequential one, continue one scan; the scratch grows
    for a longer call; resetting returns to W0."""
    spec = workloads.scaled(workloads.INPLACE_4B, T=768, C=128, d=256, f=384, seed=7)
    x = workloads.inplace_inputs(spec, device="cuda")
    Oref, Wref = ora.inplace_scan(x["Z"].cpu(), x["Vhat"].cpu(), x["W0"].cpu(), spec.eta, spec.C)
    d = spec.d
    s = cwl.FastWeightState(cwl.config("inplace", io_dtype=1, d_key=spec.f, d_val=d, chunk=128, eta=spec.eta),
                            x["W0"])
    s.set_option(cwl.abi.TTT_OPT_INPLACE_PREFIX, 1)
    O = torch.empty((spec.T, d), device="cuda", dtype=torch.bfloat16)
    s.chunk_scan(x["Z"][:128], x["Vhat"][:128], out=O[:128])      # one chunk
    s.chunk_scan(x["Z"][128:512], x["Vhat"][128:512], out=O[128:512])  # three chunks: scratch grows
    s.set_option(cwl.abi.TTT_OPT_INPLACE_PREFIX, 0)
    s.chunk_scan(x["Z"][512:], x["Vhat"][512:], out=O[512:])      # sequential form
    W = torch.empty_like(x["W0"])
    s.get_weights(W)
    torch.cuda.synchronize()
    s.poll()
    assert rel_err(O, Oref) <= TOL and rel_err(W, Wref) <= TOL
    s.reset()
    W0b = torch.empty_like(W)
    s.get_weights(W0b)
    torch.cuda.synchronize()
    assert torch.equal(W0b, x["W0"])


def test_option_rejected_for_other_states(cwl):
    from chunked_weight_layers_b200 import TTTError, abi
    W0 = torch.eye(64, device="cuda").expand(1, 2, 64, 64).contiguous()
    lin = cwl.FastWeightState(cwl.config("linear", batch=1, heads=2, chunk=16), W0)
    with pytest.raises(TTTError) as e:
        lin.set_option(abi.TTT_OPT_INPLACE_PREFIX, 1)
    assert e.value.status == abi.TTT_ERR_UNSUPPORTED


ROWS = [0, 1, 127, 128, 1000, 2047, 2048, 2559]


@pytest.mark.slow
def test_inplace_4b_workload_sampled(cwl):
    """The 4B-class workload (T=32768, d=2560, f=9728, 32 chunks) in the context-parallel form:
    sampled Wdown rows against the oracle (rows evolve independently)."""
    spec = workloads.INPLACE_4B
    x = workloads.inplace_inputs(spec, device="cuda")
    O, W, _ = scan(cwl, x, spec.C, spec.eta)
    Oref, Wref = ora.inplace_scan_rows(x["Z"].cpu(), x["Vhat"][:, ROWS].cpu(), x["W0"][ROWS].cpu(), spec.eta,
                                       spec.C)
    eo, ew = rel_err(O[:, ROWS], Oref), rel_err(W[ROWS], Wref)
    print(f"context-parallel 4B-class sampled rows: O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL
    assert torch.isfinite(O.float()).all()
